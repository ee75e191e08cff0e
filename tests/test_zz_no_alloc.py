"""attn_bwd_noalloc: the backward for callers that cannot allocate device memory.

Such callers (a custom-op or plugin interface that passes tensors but no allocator or workspace; a fixed
memory plan that forbids cudaMalloc/cudaFree, and the synchronisation they can cause, during a step) call
attn_bwd_noalloc, which takes its scratch from an array built into the library instead of a caller buffer.
These tests call it through the C ABI, on two calls in a row with different inputs and sizes (so that whatever
one call leaves in the shared array cannot leak into the next), and require:

  * dK and dV bit for bit equal to attn_bwd's (the entry point with a caller workspace): both run the same
    kernels on the same inputs, and each key tile's dK, dV accumulate in one CTA in a fixed order;
  * dQ equal to attn_bwd's up to one bf16 rounding step: dQ sums the partial products of many key tiles with
    asynchronous reductions whose order between CTAs is not fixed, so the fp32 sum can differ in its last
    bits, and after rounding to bf16 an element can land one step (2^-8 relative) away;
  * dQ, dK, dV within the parity tolerance of the float64 oracle on the second call.

This file is collected last and needs nothing from the other test files, so it also passes on its own in a
fresh process.
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


def run_both(lib, w, oracle=False):
    dev = torch.device("cuda")
    q, k, v, do = make_inputs(w)
    qd, kd, vd, dod = (x.to(dev) for x in (q, k, v, do))
    o, lse = attn.attn_fwd(qd, kd, vd, w.scale)
    ref = attn.attn_bwd(qd, kd, vd, o, lse, dod, w.scale)  # entry point with a caller workspace
    got = [torch.full_like(qd, float("nan")) for _ in range(3)]  # poisoned outputs: must all be overwritten
    stream = torch.cuda.current_stream().cuda_stream
    st = lib.attn_bwd_noalloc(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(), lse.data_ptr(),
                              dod.data_ptr(), got[0].data_ptr(), got[1].data_ptr(), got[2].data_ptr(), w.B, w.H, w.T,
                              w.D, w.scale, stream)
    assert st == 0, f"attn_bwd_noalloc: {attn._STATUS.get(st, st)} {lib.attn_last_cuda_error().decode()}"
    torch.cuda.synchronize()
    assert attn.get_device_error() == 0
    for name, g in zip(("dQ", "dK", "dV"), got):
        assert bool(torch.isfinite(g.float()).all()), f"{w.name} {name}: not fully written"
    for name, g, r in zip(("dK", "dV"), got[1:], ref[1:]):
        assert torch.equal(g, r), f"{w.name} {name}: differs from attn_bwd"
    a, b = got[0].double(), ref[0].double()
    bound = 2.0 ** -7 * b.abs() + 1e-6 * b.abs().max()
    assert bool(((a - b).abs() <= bound).all()), f"{w.name} dQ: differs from attn_bwd by more than a bf16 step"
    if oracle:
        from oracle import attn_ref
        dQ, dK, dV, _ = attn_ref.attention_backward(q, k, v, do, w.scale)
        for name, g, r in zip(("dQ", "dK", "dV"), got, (dQ, dK, dV)):
            err = np.linalg.norm(g.detach().cpu().double().numpy() - r) / np.linalg.norm(r)
            assert err <= GRAD_FRO, f"{w.name} {name}: relative Frobenius error {err:.3e} vs the oracle"


def test_noalloc_matches_workspace_entry_point_twice():
    attn_build.build()
    lib = attn.load_library()
    run_both(lib, Workload("noalloc-1", B=2, H=3, T=1000, seed=31))   # 6144 padded rows
    run_both(lib, Workload("noalloc-2", B=1, H=4, T=700, seed=32), oracle=True)  # second call: other sizes


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
