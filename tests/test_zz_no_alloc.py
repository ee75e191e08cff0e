"""attn_bwd_noalloc: the backward for callers that cannot allocate device memory.

Such callers (a custom-op or plugin interface that passes tensors but no allocator or workspace; a fixed
memory plan that forbids cudaMalloc/cudaFree, and the synchronisation they can cause, during a step) call
attn_bwd_noalloc, which takes its scratch from an array built into the library instead of a caller buffer.
These tests call it through the C ABI and require the same results as attn_bwd (the entry point with a
caller workspace), within the parity tolerance, on two calls in a row with different inputs and sizes, so
that whatever one call leaves in the shared array cannot leak into the next. This file is collected last
and needs nothing from the other test files, so it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import causal_self_attention_bf16_b200 as attn
from causal_self_attention_bf16_b200 import build as attn_build
from workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu

GRAD_FRO = 2e-2  # the parity tolerance for dQ, dK, dV


def rel_fro(a, b):
    a = a.detach().to("cpu", torch.float64).numpy()
    b = b.detach().to("cpu", torch.float64).numpy()
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)


def run_both(lib, w):
    dev = torch.device("cuda")
    q, k, v, do = (x.to(dev) for x in make_inputs(w))
    o, lse = attn.attn_fwd(q, k, v, w.scale)
    ref = attn.attn_bwd(q, k, v, o, lse, do, w.scale)  # entry point with a caller workspace
    got = [torch.full_like(q, float("nan")) for _ in range(3)]  # poisoned outputs: must all be overwritten
    stream = torch.cuda.current_stream().cuda_stream
    st = lib.attn_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                              got[0].data_ptr(), got[1].data_ptr(), got[2].data_ptr(), w.B, w.H, w.T, w.D, w.scale,
                              stream)
    assert st == 0, f"attn_bwd_noalloc: {attn._STATUS.get(st, st)} {lib.attn_last_cuda_error().decode()}"
    torch.cuda.synchronize()
    assert attn.get_device_error() == 0
    for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
        assert bool(torch.isfinite(g.float()).all()), f"{name}: not fully written"
        err = rel_fro(g, r)
        assert err <= GRAD_FRO, f"{w.name} {name}: relative Frobenius error {err:.3e} vs attn_bwd"


def test_noalloc_matches_workspace_entry_point_twice():
    attn_build.build()
    lib = attn.load_library()
    run_both(lib, Workload("noalloc-1", B=2, H=3, T=1000, seed=31))   # 6144 padded rows
    run_both(lib, Workload("noalloc-2", B=1, H=4, T=700, seed=32))    # second call: other sizes and inputs


def test_noalloc_rejects_sizes_beyond_its_array():
    lib = attn.load_library()
    dev = torch.device("cuda")
    q = torch.zeros(1, 128, 1, 128, dtype=torch.bfloat16, device=dev)
    lse = torch.zeros(1, 1, 128, dtype=torch.float32, device=dev)
    outs = [torch.empty_like(q) for _ in range(3)]
    # 64 * 8 * roundup(2048) = 1,048,576 rows: far beyond the 64512 the array holds. Checked before any launch
    # (the pointers are never read for these sizes).
    st = lib.attn_bwd_noalloc(q.data_ptr(), q.data_ptr(), q.data_ptr(), q.data_ptr(), lse.data_ptr(), q.data_ptr(),
                              outs[0].data_ptr(), outs[1].data_ptr(), outs[2].data_ptr(), 64, 8, 2048, 128, 0.088,
                              None)
    assert st == 6  # ATTN_ERR_WORKSPACE
    assert "scratch" in lib.attn_last_cuda_error().decode()
