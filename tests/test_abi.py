"""The C-ABI library loads, exports every symbol include/attn.h declares, and validates arguments on the host.

No test here needs a GPU: argument errors are detected before any CUDA call, and a well-formed call on a
machine without an sm_100 device must fail loudly (ATTN_ERR_CUDA), never fall back to a CPU path.
"""
import ctypes
import os
import re

import pytest
import torch

import causal_self_attention_bf16_b200 as attn
from causal_self_attention_bf16_b200 import build as attn_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


@pytest.fixture(scope="module")
def lib():
    attn_build.build()
    return attn.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("attn_fwd", "attn_bwd", "attn_bwd_workspace_bytes", "attn_status_string"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert names, "no declarations parsed"
    for n in names:
        assert hasattr(lib, n), f"libattn.so does not export {n}"
    assert set(names) == set(attn.SIGNATURES), "binding signature table and header disagree"


def test_abi_version_and_status_strings(lib):
    assert lib.attn_abi_version() == 2
    for code, name in attn._STATUS.items():
        assert lib.attn_status_string(code).decode() == name


def test_workspace_size_formula(lib):
    # lse2 + delta: B*H*Tp fp32 each (256-byte rounded), accumulator B*H*Tp*128 fp32.
    for B, H, T in ((1, 1, 1), (2, 3, 100), (32, 10, 2048)):
        Tp = (T + 127) // 128 * 128
        rows = B * H * Tp
        up = lambda x: (x + 255) // 256 * 256
        assert lib.attn_bwd_workspace_bytes(B, H, T, 128) == 2 * up(rows * 4) + up(rows * 512)
    assert lib.attn_bwd_workspace_bytes(1, 1, 1, 64) == 0
    assert lib.attn_bwd_workspace_bytes(0, 1, 1, 128) == 0


# Fake, aligned, non-overlapping device addresses: never dereferenced on the host, and every call below
# fails its checks before anything reaches CUDA.
def fake_ptrs(n, size):
    base = 1 << 40
    return [base + i * (size + (1 << 20)) for i in range(n)]


def fwd_call(lib, q, k, v, o, lse, B=1, H=2, T=128, D=128, scale=0.088):
    return lib.attn_fwd(q, k, v, o, lse, B, H, T, D, scale, None)


def test_fwd_argument_errors(lib):
    size = 1 * 128 * 2 * 128 * 2
    q, k, v, o, lse = fake_ptrs(5, size)
    assert fwd_call(lib, None, k, v, o, lse) == 1
    assert fwd_call(lib, q, k, v, None, lse) == 1
    assert fwd_call(lib, q, k, v, o, lse, B=0) == 1
    assert fwd_call(lib, q, k, v, o, lse, T=-3) == 1
    assert fwd_call(lib, q, k, v, o, lse, scale=0.0) == 1
    assert fwd_call(lib, q, k, v, o, lse, scale=float("nan")) == 1
    assert fwd_call(lib, q, k, v, o, lse, scale=float("inf")) == 1
    assert fwd_call(lib, q, k, v, o, lse, D=64) == 2
    assert fwd_call(lib, q + 8, k, v, o, lse) == 3
    assert fwd_call(lib, q, k, v, o, lse + 4) == 3
    assert fwd_call(lib, q, k, v, q + 256, lse) == 1          # o overlaps q
    assert fwd_call(lib, q, k, v, o, o + 1024) == 1           # lse overlaps o


def bwd_call(lib, ptrs, ws_bytes, B=1, H=2, T=128, D=128, scale=0.088, **over):
    names = ["q", "k", "v", "o", "lse", "dO", "dq", "dk", "dv", "ws"]
    args = dict(zip(names, ptrs))
    args.update(over)
    return lib.attn_bwd(*[args[n] for n in names], ws_bytes, B, H, T, D, scale, None)


def test_bwd_argument_errors(lib):
    size = 1 * 128 * 2 * 128 * 2
    ws = lib.attn_bwd_workspace_bytes(1, 2, 128, 128)
    ptrs = fake_ptrs(10, max(size, ws))
    assert bwd_call(lib, ptrs, ws, dq=None) == 1
    assert bwd_call(lib, ptrs, ws, D=96) == 2
    assert bwd_call(lib, ptrs, ws - 1) == 6
    assert bwd_call(lib, ptrs, ws, ws=None) == 6
    assert bwd_call(lib, ptrs, ws, dk=ptrs[7] + 8) == 3
    assert bwd_call(lib, ptrs, ws, ws=ptrs[9] + 16) == 3      # workspace must be 256-byte aligned
    assert bwd_call(lib, ptrs, ws, dq=ptrs[0]) == 1           # dq aliases q
    assert bwd_call(lib, ptrs, ws, dv=ptrs[6]) == 1           # dv aliases dq
    assert bwd_call(lib, ptrs, ws, ws=ptrs[8]) == 1           # workspace aliases dv


def test_gqa_argument_errors(lib):
    """attn_fwd_gqa / attn_bwd_gqa reject key/value head counts that do not divide H, and check overlaps with
    the k, v, dk, dv sizes of H_kv heads."""
    qsize = 1 * 128 * 6 * 128 * 2
    q, k, v, o, lse = fake_ptrs(5, qsize)
    for hkv in (0, 4, 7, -2):
        assert lib.attn_fwd_gqa(q, k, v, o, lse, 1, 6, hkv, 128, 128, 0.088, None) == 1
    assert lib.attn_fwd_gqa(q, k, v, o, lse, 1, 6, 3, 128, 96, 0.088, None) == 2
    assert lib.attn_fwd_gqa(q, k, v, k + 256, lse, 1, 6, 3, 128, 128, 0.088, None) == 1   # o overlaps k
    ws = lib.attn_bwd_workspace_bytes(1, 6, 128, 128)
    ptrs = fake_ptrs(10, max(qsize, ws))
    args = lambda **over: [over.get(n, p) for n, p in zip(["q", "k", "v", "o", "lse", "dO", "dq", "dk", "dv", "ws"], ptrs)]
    assert lib.attn_bwd_gqa(*args(), ws, 1, 6, 4, 128, 128, 0.088, None) == 1
    assert lib.attn_bwd_gqa(*args(), ws - 1, 1, 6, 2, 128, 128, 0.088, None) == 6
    assert lib.attn_bwd_gqa(*args(dk=ptrs[1]), ws, 1, 6, 2, 128, 128, 0.088, None) == 1    # dk aliases k


def test_window_argument_errors(lib):
    """attn_fwd_ex / attn_bwd_ex take window >= 0, or -1 for none; anything below is an argument error."""
    qsize = 1 * 128 * 2 * 128 * 2
    q, k, v, o, lse = fake_ptrs(5, qsize)
    for w in (-2, -100):
        assert lib.attn_fwd_ex(q, k, v, o, lse, 1, 2, 2, 128, 128, 0.088, w, None) == 1
    assert lib.attn_fwd_ex(q, k, v, o, lse, 1, 2, 3, 128, 128, 0.088, 5, None) == 1  # H_kv does not divide H
    ws = lib.attn_bwd_workspace_bytes(1, 2, 128, 128)
    ptrs = fake_ptrs(10, max(qsize, ws))
    assert lib.attn_bwd_ex(*ptrs, ws, 1, 2, 2, 128, 128, 0.088, -2, None) == 1
    assert lib.attn_bwd_ex(*ptrs, ws - 1, 1, 2, 2, 128, 128, 0.088, 4, None) == 6


def test_decode_split_rule(lib):
    """The cache is split into about 4 CTAs per SM of a 148-SM part, in chunks of at least 256 keys that are whole
    128-key blocks; the workspace holds each chunk's unnormalised O (128 floats) and its max and sum per row."""
    row = (128 + 2) * 4
    assert lib.attn_decode_workspace_bytes(64, 10, 10, 1, 2048, 128) == 640 * 1 * 1 * row  # 640 pairs: no split
    assert lib.attn_decode_workspace_bytes(64, 10, 5, 1, 2048, 128) == 320 * 2 * 2 * row   # 320 pairs: 2 chunks
    assert lib.attn_decode_workspace_bytes(2, 8, 2, 1, 1000, 128) == 4 * 4 * 4 * row      # 4 chunks of 256 keys
    assert lib.attn_decode_workspace_bytes(1, 1, 1, 1, 100, 128) == 1 * row               # shorter than a chunk


def test_decode_kernel_count(lib):
    """One kernel when each (sequence, head) is one chunk of the cache (it writes o and lse itself), two when the
    chunks are merged by a second kernel; 0 for arguments attn_decode_ex rejects."""
    assert lib.attn_decode_kernels(64, 10, 10, 1, 2048, 128, -1) == 1   # 640 pairs: no split
    assert lib.attn_decode_kernels(64, 10, 5, 1, 2048, 128, -1) == 2    # 320 pairs: 2 chunks
    assert lib.attn_decode_kernels(64, 10, 10, 1, 2048, 128, 512) == 1  # the window's band is one chunk
    assert lib.attn_decode_kernels(4, 1, 1, 4, 5, 128, -1) == 1         # shorter than a chunk
    assert lib.attn_decode_kernels(2, 8, 3, 1, 1000, 128, -1) == 0      # H_kv does not divide H
    assert lib.attn_decode_kernels(2, 8, 2, 1, 1000, 128, -2) == 0      # window < -1


def test_decode_argument_errors(lib):
    """attn_decode checks sizes, the row limit, the workspace and overlaps before any CUDA call."""
    assert lib.attn_decode_workspace_bytes(2, 8, 2, 1, 1000, 128) > 0
    assert lib.attn_decode_workspace_bytes(2, 8, 3, 1, 1000, 128) == 0     # H_kv does not divide H
    assert lib.attn_decode_workspace_bytes(2, 64, 1, 1, 1000, 128) == 0    # 64 rows per CTA > 32
    ws = lib.attn_decode_workspace_bytes(2, 8, 2, 1, 1000, 128)
    q, kc, vc, lens, o, lse, w = fake_ptrs(7, max(2 * 1000 * 2 * 128 * 2, ws))
    call = lambda **kw: lib.attn_decode(kw.get("q", q), kc, vc, kw.get("lens", lens), kw.get("o", o), lse,
                                        kw.get("w", w), kw.get("wb", ws), 2, 8, kw.get("hkv", 2), 1, 1000,
                                        kw.get("D", 128), 0.088, None)
    assert call(q=None) == 1
    assert call(hkv=3) == 1
    assert call(D=64) == 2
    assert call(wb=ws - 1) == 6
    assert call(o=q) == 1                 # o aliases q
    assert call(w=kc) == 1                # workspace aliases the cache
    assert call(lens=lens + 2) == 3       # lengths must be 4-byte aligned


def test_qk_norm_rope_argument_errors(lib):
    """The prologue checks sizes, base, eps, pairing, alignment and overlaps before any CUDA call; in place
    (an output equal to its input) is allowed, a partial overlap is not."""
    B, T, H, Hkv = 2, 100, 4, 2
    qb, kb = B * T * H * 256, B * T * Hkv * 256
    q, k, qo, ko, offs, gq, gk = fake_ptrs(7, qb)
    fwd = lambda **kw: lib.attn_qk_norm_rope(kw.get("q", q), k, kw.get("qo", qo), kw.get("ko", ko),
                                             kw.get("offs", offs), B, kw.get("T", T), H, kw.get("hkv", Hkv),
                                             kw.get("D", 128), kw.get("base", 10000.0), kw.get("eps", 1e-6),
                                             kw.get("pairing", 0), None)
    assert fwd(q=None) == 1
    assert fwd(T=0) == 1 and fwd(hkv=0) == 1
    assert fwd(D=64) == 2
    assert fwd(base=0.0) == 1 and fwd(base=float("inf")) == 1 and fwd(base=-2.0) == 1
    assert fwd(eps=-1e-6) == 1 and fwd(eps=float("nan")) == 1
    assert fwd(pairing=2) == 1 and fwd(pairing=-1) == 1
    assert fwd(qo=qo + 8) == 3
    assert fwd(offs=offs + 2) == 3
    assert fwd(qo=q + 256) == 1           # output overlaps its input without being it
    assert fwd(qo=k) == 1                 # q's output over k
    assert fwd(ko=qo + qb - 256) == 1     # the two outputs overlap
    assert fwd(offs=qo) == 1              # positions inside an output
    bwd = lambda **kw: lib.attn_qk_norm_rope_bwd(q, k, kw.get("gq", gq), gk, kw.get("dq", qo), kw.get("dk", ko),
                                                 None, B, T, H, Hkv, 128, 10000.0, 1e-6, kw.get("pairing", 1), None)
    assert bwd(dq=q) == 1                 # dq over the input q
    assert bwd(dq=gq + 256) == 1          # partial overlap with its own gradient
    assert bwd(dq=gk) == 1                # dq over dk_out
    assert bwd(pairing=5) == 1


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_no_cpu_fallback_without_gpu(lib):
    """A well-formed call on a machine without an sm_100 GPU fails loudly instead of computing on the CPU."""
    size = 1 * 128 * 2 * 128 * 2
    q, k, v, o, lse = fake_ptrs(5, size)
    assert fwd_call(lib, q, k, v, o, lse) == 4
    assert lib.attn_last_cuda_error().decode() != ""
    ws = lib.attn_bwd_workspace_bytes(1, 2, 128, 128)
    assert bwd_call(lib, fake_ptrs(10, max(size, ws)), ws) == 4
    assert lib.attn_fwd_gqa(q, k, v, o, lse, 1, 2, 1, 128, 128, 0.088, None) == 4
    # the prologue: in place is well formed, and still fails loudly
    assert lib.attn_qk_norm_rope(q, k, q, k, None, 1, 128, 2, 2, 128, 10000.0, 1e-6, 0, None) == 4
    assert lib.attn_last_cuda_error().decode() != ""
    assert lib.attn_qk_norm_rope_bwd(q, k, o, lse, o, lse, None, 1, 128, 2, 2, 128, 10000.0, 1e-6, 1, None) == 4


def test_binding_rejects_cpu_tensors(lib):
    q = torch.zeros(1, 128, 2, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        attn.attn_fwd(q, q, q)


def test_binding_signatures_match_header_argument_counts():
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    for name, (argtypes, _) in attn.SIGNATURES.items():
        m = re.search(name + r"\s*\(([^)]*)\)", text)
        assert m, name
        params = [p for p in m.group(1).split(",") if p.strip() and p.strip() != "void"]
        assert len(params) == len(argtypes), f"{name}: header has {len(params)} params, binding {len(argtypes)}"


def test_binding_checks_every_backward_buffer():
    """The backward wrappers (attn_bwd and attn_bwd_noalloc share one check) reject an lse of the wrong dtype,
    shape or layout and a gradient buffer of the wrong shape: the kernels read and write whole tensors, so a
    smaller buffer would be written past its end."""
    B, T, H, D = 1, 16, 2, 128
    q = torch.zeros(B, T, H, D, dtype=torch.bfloat16)
    lse = torch.zeros(B, H, T, dtype=torch.float32)
    dq, dk, dv, hkv = attn._bwd_tensors(q, q, q, q, lse, q, None, None, None, same_heads=True)
    assert dq.shape == q.shape and hkv == H
    bad_lse = [lse.to(torch.bfloat16), torch.zeros(B, H, T - 1), torch.zeros(B, T, H).transpose(1, 2)]
    for bad in bad_lse:
        with pytest.raises(ValueError):
            attn._bwd_tensors(q, q, q, q, bad, q, None, None, None, same_heads=True)
        with pytest.raises(ValueError):
            attn._fwd_tensors(q, q, q, None, bad)
    small = torch.zeros(B, T - 1, H, D, dtype=torch.bfloat16)
    for pos in range(3):
        grads = [None, None, None]
        grads[pos] = small
        with pytest.raises(ValueError):
            attn._bwd_tensors(q, q, q, q, lse, q, *grads, same_heads=True)
    # same_heads (the allocation-free form has no key/value head count): fewer key/value heads are rejected
    kv = torch.zeros(B, T, 1, D, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        attn._bwd_tensors(q, kv, kv, q, lse, q, None, None, None, same_heads=True)
    assert attn._bwd_tensors(q, kv, kv, q, lse, q, None, None, None)[3] == 1


def test_binding_rejects_tensors_on_different_devices():
    B, T, H, D = 1, 16, 2, 128
    q = torch.zeros(B, T, H, D, dtype=torch.bfloat16)
    other = torch.zeros(B, T, H, D, dtype=torch.bfloat16, device="meta")
    lse = torch.zeros(B, H, T, dtype=torch.float32)
    with pytest.raises(ValueError, match="one call"):
        attn._bwd_tensors(q, other, q, q, lse, q, None, None, None)
    with pytest.raises(ValueError, match="one call"):
        attn._bwd_tensors(q, q, q, q, lse.to("meta"), q, None, None, None)
    with pytest.raises(ValueError, match="one call"):
        attn._fwd_tensors(q, q, other, None, None)
