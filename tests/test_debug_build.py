"""The debug build (libattn_debug.so, -DATTN_DEBUG): the same kernels with every plain-address access checked.

CPU: both builds load with every declared symbol and tell which they are; the release build refuses the bounds
self-test before touching the GPU. GPU: the self-test's checked store past its array's declared extent records
exactly its site (kind 2) and writes nothing; every kind of call (forward, backward in stages, grouped heads and
a window, ragged lengths, cached decode with and without a window, the prologue forward and backward) gives the
release build's results through the debug build with a clean error word, so no check fires on valid inputs.
"""
import ctypes
import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import causal_self_attention_bf16_b200 as attn  # noqa: E402
from causal_self_attention_bf16_b200 import build as attn_build  # noqa: E402

SITE_SELFTEST = 0x7E
KIND_BOUNDS = 2


@pytest.fixture(scope="module")
def libs():
    release = attn.open_library(attn_build.build())
    debug = attn.open_library(attn_build.build(debug=True))
    return release, debug


def test_both_builds_load_and_say_which_they_are(libs):
    release, debug = libs
    assert release.attn_is_debug_build() == 0
    assert debug.attn_is_debug_build() == 1
    assert release.attn_abi_version() == debug.attn_abi_version()
    assert debug.attn_status_string(7) == b"ATTN_ERR_BOUNDS"


def test_release_build_refuses_the_bounds_selftest(libs):
    release, _ = libs
    assert release.attn_selftest_bounds_check(None) == 2  # ATTN_ERR_UNSUPPORTED, before any CUDA call


def _error_word(lib):
    w = ctypes.c_uint32(0)
    st = lib.attn_get_device_error(ctypes.byref(w))
    return st, int(w.value)


@pytest.mark.gpu
def test_bounds_selftest_records_its_site_and_skips_the_store(libs):
    _, debug = libs
    assert debug.attn_clear_device_error() == 0
    assert debug.attn_selftest_bounds_check(None) == 0
    st, word = _error_word(debug)
    assert st == 7 and word == (SITE_SELFTEST << 8) | KIND_BOUNDS, hex(word)
    assert debug.attn_clear_device_error() == 0
    assert _error_word(debug) == (0, 0)


def _fwd_bwd(lib, q, k, v, do, H, Hkv, window, scale):
    B, T = q.shape[0], q.shape[1]
    s = torch.cuda.current_stream().cuda_stream
    o = torch.empty_like(q)
    lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    assert lib.attn_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, Hkv, T,
                           128, scale, window, s) == 0
    wsb = lib.attn_bwd_workspace_bytes(B, H, T, 128)
    ws = torch.empty(wsb, dtype=torch.uint8, device=q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    assert lib.attn_bwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                           dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), wsb, B, H, Hkv, T, 128,
                           scale, window, s) == 0
    torch.cuda.synchronize()
    return o, lse, dq, dk, dv


def _decode(lib, q, kc, vc, lens, H, Hkv, window, scale):
    B, Tq, Tk = q.shape[0], q.shape[1], kc.shape[1]
    s = torch.cuda.current_stream().cuda_stream
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Tq), dtype=torch.float32, device=q.device)
    wsb = lib.attn_decode_workspace_bytes(B, H, Hkv, Tq, Tk, 128)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=q.device)
    assert lib.attn_decode_ex(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), lens.data_ptr(), o.data_ptr(),
                              lse.data_ptr(), ws.data_ptr(), wsb, B, H, Hkv, Tq, Tk, 128, scale, window, s) == 0
    torch.cuda.synchronize()
    return o, lse


def _prologue(lib, q, k, gq, gk, offsets, H, Hkv, pairing):
    B, T = q.shape[0], q.shape[1]
    s = torch.cuda.current_stream().cuda_stream
    qo, ko, dq, dk = torch.empty_like(q), torch.empty_like(k), torch.empty_like(q), torch.empty_like(k)
    off = offsets.data_ptr() if offsets is not None else None
    assert lib.attn_qk_norm_rope(q.data_ptr(), k.data_ptr(), qo.data_ptr(), ko.data_ptr(), off, B, T, H, Hkv, 128,
                                 10000.0, 1e-6, pairing, s) == 0
    assert lib.attn_qk_norm_rope_bwd(q.data_ptr(), k.data_ptr(), gq.data_ptr(), gk.data_ptr(), dq.data_ptr(),
                                     dk.data_ptr(), off, B, T, H, Hkv, 128, 10000.0, 1e-6, pairing, s) == 0
    torch.cuda.synchronize()
    return qo, ko, dq, dk


def _randn(shape, g, dev):
    return torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16).to(dev)


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,Hkv,T,window", [(1, 2, 2, 128, -1), (2, 3, 3, 129, -1), (1, 2, 2, 383, -1),
                                              (2, 4, 2, 300, -1), (1, 2, 2, 300, 100), (1, 4, 1, 1000, 129)])
def test_debug_build_matches_release_on_attention(libs, B, H, Hkv, T, window):
    release, debug = libs
    dev = torch.device("cuda:0")
    g = torch.Generator().manual_seed(1000 + T + H)
    q, do = _randn((B, T, H, 128), g, dev), _randn((B, T, H, 128), g, dev)
    k, v = _randn((B, T, Hkv, 128), g, dev), _randn((B, T, Hkv, 128), g, dev)
    scale = 128 ** -0.5
    assert debug.attn_clear_device_error() == 0
    ref = _fwd_bwd(release, q, k, v, do, H, Hkv, window, scale)
    got = _fwd_bwd(debug, q, k, v, do, H, Hkv, window, scale)
    assert _error_word(debug) == (0, 0), "an address check fired on valid inputs"
    for name, a, b in zip(("o", "lse", "dq", "dk", "dv"), ref, got):
        if name == "dq":  # the accumulation order of the bulk reductions varies from run to run
            err = (a.float() - b.float()).norm() / a.float().norm()
            assert err < 1e-2, f"dq differs: relative {err:.2e}"
        else:
            assert torch.equal(a, b), f"{name} differs between the builds"


@pytest.mark.gpu
@pytest.mark.parametrize("window,Tk,kernels", [(-1, 700, 2), (100, 700, 1), (-1, 200, 1)])
def test_debug_build_matches_release_on_decode(libs, window, Tk, kernels):
    """A split cache (chunks merged by the second kernel), and a window band or a cache short enough to be one
    chunk per (sequence, head), whose split kernel writes o and lse itself."""
    release, debug = libs
    dev = torch.device("cuda:0")
    g = torch.Generator().manual_seed(77)
    B, H, Hkv, Tq = 3, 8, 2, 2
    assert release.attn_decode_kernels(B, H, Hkv, Tq, Tk, 128, window) == kernels
    q = _randn((B, Tq, H, 128), g, dev)
    kc, vc = _randn((B, Tk, Hkv, 128), g, dev), _randn((B, Tk, Hkv, 128), g, dev)
    lens = torch.tensor([Tk, 1, Tk // 2], dtype=torch.int32, device=dev)
    assert debug.attn_clear_device_error() == 0
    ref = _decode(release, q, kc, vc, lens, H, Hkv, window, 128 ** -0.5)
    got = _decode(debug, q, kc, vc, lens, H, Hkv, window, 128 ** -0.5)
    assert _error_word(debug) == (0, 0), "an address check fired on valid inputs"
    for name, a, b in zip(("o", "lse"), ref, got):
        assert torch.equal(a, b), f"decode {name} differs between the builds"


@pytest.mark.gpu
@pytest.mark.parametrize("pairing", [0, 1])
def test_debug_build_matches_release_on_the_prologue(libs, pairing):
    release, debug = libs
    dev = torch.device("cuda:0")
    g = torch.Generator().manual_seed(5 + pairing)
    B, T, H, Hkv = 2, 37, 5, 2
    q, k = _randn((B, T, H, 128), g, dev), _randn((B, T, Hkv, 128), g, dev)
    gq, gk = _randn((B, T, H, 128), g, dev), _randn((B, T, Hkv, 128), g, dev)
    offsets = torch.tensor([0, 9000], dtype=torch.int32, device=dev)
    assert debug.attn_clear_device_error() == 0
    ref = _prologue(release, q, k, gq, gk, offsets, H, Hkv, pairing)
    got = _prologue(debug, q, k, gq, gk, offsets, H, Hkv, pairing)
    assert _error_word(debug) == (0, 0), "an address check fired on valid inputs"
    for name, a, b in zip(("q_out", "k_out", "dq", "dk"), ref, got):
        assert torch.equal(a, b), f"prologue {name} differs between the builds"
