"""Thin Python binding of libattn.so: bf16 causal multi-head self-attention, forward and backward, on B200.

Every step of the computation runs in the library's sm_100a kernels. This module only marshals arguments:
it checks dtypes/shapes, allocates outputs with torch (device memory is plumbing), and passes raw device
pointers and the current CUDA stream through the C ABI declared in include/attn.h. There is no CPU path: if
the library is missing or the device is not an sm_100 GPU, the calls raise.

The operation is nanochat's ``flash_attn_func(q, k, v, causal=True)`` on [B, T, H, D] tensors (apidog "Train
your own ChatGPT", section 5 "Flash Attention integration"), with the textbook definition written out in
include/attn.h.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG_DIR, "libattn.so")
DEBUG_LIB_PATH = os.path.join(_PKG_DIR, "libattn_debug.so")  # the same sources with address checks

ATTN_OK = 0
_STATUS = {0: "ATTN_OK", 1: "ATTN_ERR_INVALID_ARG", 2: "ATTN_ERR_UNSUPPORTED", 3: "ATTN_ERR_MISALIGNED",
           4: "ATTN_ERR_CUDA", 5: "ATTN_ERR_TIMEOUT", 6: "ATTN_ERR_WORKSPACE", 7: "ATTN_ERR_BOUNDS"}

# Exported symbols of the C ABI (include/attn.h), with their ctypes signatures.
_VP, _I, _F, _SZ, _U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_uint64
SIGNATURES = {
    "attn_abi_version": ([], _I),
    "attn_status_string": ([_I], ctypes.c_char_p),
    "attn_last_cuda_error": ([], ctypes.c_char_p),
    "attn_fwd": ([_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _F, _VP], _I),
    "attn_bwd_workspace_bytes": ([_I, _I, _I, _I], _SZ),
    "attn_bwd": ([_VP] * 10 + [_SZ, _I, _I, _I, _I, _F, _VP], _I),
    "attn_bwd_preprocess": ([_VP] * 10 + [_SZ, _I, _I, _I, _I, _F, _VP], _I),
    "attn_bwd_dkdv": ([_VP] * 10 + [_SZ, _I, _I, _I, _I, _F, _VP], _I),
    "attn_bwd_dq_convert": ([_VP] * 10 + [_SZ, _I, _I, _I, _I, _F, _VP], _I),
    "attn_bwd_noalloc": ([_VP] * 9 + [_I, _I, _I, _I, _F, _VP], _I),
    "attn_fwd_gqa": ([_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _F, _VP], _I),
    "attn_bwd_gqa": ([_VP] * 10 + [_SZ, _I, _I, _I, _I, _I, _F, _VP], _I),
    "attn_fwd_ex": ([_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _F, _I, _VP], _I),
    "attn_bwd_ex": ([_VP] * 10 + [_SZ, _I, _I, _I, _I, _I, _F, _I, _VP], _I),
    "attn_decode_workspace_bytes": ([_I] * 6, _SZ),
    "attn_decode_kernels": ([_I] * 7, _I),
    "attn_decode": ([_VP] * 7 + [_SZ] + [_I] * 6 + [_F, _VP], _I),
    "attn_decode_ex": ([_VP] * 7 + [_SZ] + [_I] * 6 + [_F, _I, _VP], _I),
    "attn_qk_norm_rope": ([_VP] * 5 + [_I] * 5 + [_F, _F, _I, _VP], _I),
    "attn_qk_norm_rope_bwd": ([_VP] * 7 + [_I] * 5 + [_F, _F, _I, _VP], _I),
    "attn_get_device_error": ([ctypes.POINTER(ctypes.c_uint32)], _I),
    "attn_clear_device_error": ([], _I),
    "attn_set_wait_limit_ns": ([_U64], _I),
    "attn_selftest_wait_timeout": ([_U64, _VP], _I),
    "attn_is_debug_build": ([], _I),
    "attn_selftest_bounds_check": ([_VP], _I),
}


class AttnError(RuntimeError):
    """A non-OK status returned by libattn.so."""

    def __init__(self, fn: str, status: int, detail: str = ""):
        self.status = status
        msg = f"{fn} returned {_STATUS.get(status, status)}"
        if detail:
            msg += f" ({detail})"
        super().__init__(msg)


_lib = None


def open_library(path: str) -> ctypes.CDLL:
    """Open a build of the library (libattn.so or libattn_debug.so) with the C signatures attached."""
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m causal_self_attention_bf16_b200.build` "
                          "(--debug for libattn_debug.so, or __graft_entry__.build()); there is no fallback "
                          "implementation")
    lib = ctypes.CDLL(path)
    for name, (argtypes, restype) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.argtypes = argtypes
        fn.restype = restype
    return lib


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """The library every function of this package calls, loaded once: libattn.so, or libattn_debug.so (the
    address-checking build) when the environment sets ATTN_LIBRARY=debug. Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if path is None:
        path = DEBUG_LIB_PATH if os.environ.get("ATTN_LIBRARY") == "debug" else LIB_PATH
    _lib = open_library(path)
    return _lib


def _check(fn: str, status: int):
    if status != ATTN_OK:
        detail = ""
        if status == 4:
            lib = load_library()
            detail = lib.attn_last_cuda_error().decode(errors="replace")
        raise AttnError(fn, status, detail)


def _stream_handle(stream: Optional[torch.cuda.Stream], device: torch.device) -> int:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return s.cuda_stream


def _require_cuda(name: str, t) -> None:
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")


def _check_qkv(name: str, t: torch.Tensor, shape=None, device: Optional[torch.device] = None):
    """A bf16, contiguous, 4-D tensor (of `shape`, on `device`, where given)."""
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name} must be a tensor")
    if t.dtype != torch.bfloat16:
        raise ValueError(f"{name} must be bfloat16, got {t.dtype}")
    if t.dim() != 4 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous [B, T, H, D] tensor")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}; every tensor of one call must be on {device}")


def _check_f32(name: str, t: torch.Tensor, shape, device: torch.device):
    """A contiguous fp32 tensor of `shape` on `device` (lse)."""
    if (not isinstance(t, torch.Tensor) or t.dtype != torch.float32 or tuple(t.shape) != tuple(shape)
            or not t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous fp32 {list(shape)} tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}; every tensor of one call must be on {device}")


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)


def _kv_shape(q: torch.Tensor, k: torch.Tensor):
    """[B, T, H_kv, D] of k and v: H_kv = H, or fewer key/value heads dividing H (grouped-query attention)."""
    _check_qkv("k", k, device=q.device)
    B, T, H, D = q.shape
    Hkv = k.shape[2]
    if (k.shape[0], k.shape[1], k.shape[3]) != (B, T, D) or Hkv < 1 or H % Hkv:
        raise ValueError(f"k has shape {tuple(k.shape)}; expected [{B}, {T}, H_kv, {D}] with H_kv dividing {H}")
    return (B, T, Hkv, D)


def _fwd_tensors(q, k, v, o, lse):
    """Check the forward's tensors (all on q's device) and allocate the outputs not given. Returns
    (o, lse, H_kv)."""
    _check_qkv("q", q)
    B, T, H, D = q.shape
    kv = _kv_shape(q, k)
    _check_qkv("v", v, kv, q.device)
    o = torch.empty_like(q) if o is None else o
    _check_qkv("o", o, q.shape, q.device)
    if lse is None:
        lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    _check_f32("lse", lse, (B, H, T), q.device)
    return o, lse, kv[2]


def _bwd_tensors(q, k, v, o, lse, dO, dq, dk, dv, same_heads: bool = False):
    """Check the backward's tensors (all on q's device; with same_heads, k and v must have q's shape) and
    allocate the gradients not given. The kernels read and write whole tensors of these shapes, so every
    caller-supplied buffer is checked here: a smaller one would be written past its end. Returns
    (dq, dk, dv, H_kv)."""
    _check_qkv("q", q)
    B, T, H, D = q.shape
    dev = q.device
    if same_heads:
        _check_qkv("k", k, q.shape, dev)
        kv = tuple(q.shape)
    else:
        kv = _kv_shape(q, k)
    _check_qkv("v", v, kv, dev)
    for name, t in (("o", o), ("dO", dO)):
        _check_qkv(name, t, q.shape, dev)
    _check_f32("lse", lse, (B, H, T), dev)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check_qkv("dq", dq, q.shape, dev)
    _check_qkv("dk", dk, kv, dev)
    _check_qkv("dv", dv, kv, dev)
    return dq, dk, dv, kv[2]


def _window_arg(window: Optional[int]) -> int:
    if window is None:
        return -1
    if int(window) < 0:
        raise ValueError("window must be >= 0 (or None for no window)")
    return int(window)


def attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: Optional[float] = None,
             o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
             stream: Optional[torch.cuda.Stream] = None, window: Optional[int] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Causal attention forward. q: bf16 [B, T, H, D]; k, v: bf16 [B, T, H_kv, D] with H_kv = H, or H_kv
    dividing H for grouped-query attention (query head h reads key/value head h // (H // H_kv)); all on one
    CUDA device. window: None, or a sliding window (query i sees keys i - window .. i). Returns
    (o [B, T, H, D], lse [B, H, T])."""
    lib = load_library()
    _require_cuda("q", q)
    o, lse, Hkv = _fwd_tensors(q, k, v, o, lse)
    B, T, H, D = q.shape
    scale = default_scale(D) if scale is None else float(scale)
    win = _window_arg(window)
    with torch.cuda.device(q.device):
        sh = _stream_handle(stream, q.device)
        if win >= 0:
            st = lib.attn_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, Hkv,
                                 T, D, scale, win, sh)
            _check("attn_fwd_ex", st)
        elif Hkv == H:
            st = lib.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, T, D,
                              scale, sh)
            _check("attn_fwd", st)
        else:
            st = lib.attn_fwd_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, Hkv,
                                  T, D, scale, sh)
            _check("attn_fwd_gqa", st)
    return o, lse


def attn_bwd_workspace_bytes(B: int, H: int, T: int, D: int) -> int:
    return int(load_library().attn_bwd_workspace_bytes(B, H, T, D))


def attn_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor,
             dO: torch.Tensor, scale: Optional[float] = None, dq: Optional[torch.Tensor] = None,
             dk: Optional[torch.Tensor] = None, dv: Optional[torch.Tensor] = None,
             workspace: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None,
             window: Optional[int] = None):
    """Causal attention backward (window as given to attn_fwd). Returns (dq [B, T, H, D], dk, dv [B, T, H_kv,
    D]); with grouped-query
    attention dk, dv are the gradients of the shared heads (summed over each group's query heads)."""
    lib = load_library()
    _require_cuda("q", q)
    dq, dk, dv, Hkv = _bwd_tensors(q, k, v, o, lse, dO, dq, dk, dv)
    B, T, H, D = q.shape
    need = attn_bwd_workspace_bytes(B, H, T, D)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    elif workspace.device != q.device:
        raise ValueError(f"workspace is on {workspace.device}; every tensor of one call must be on {q.device}")
    scale = default_scale(D) if scale is None else float(scale)
    ptrs = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), dO.data_ptr(), dq.data_ptr(),
            dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(), workspace.numel() * workspace.element_size())
    win = _window_arg(window)
    with torch.cuda.device(q.device):
        sh = _stream_handle(stream, q.device)
        if win >= 0:
            st = lib.attn_bwd_ex(*ptrs, B, H, Hkv, T, D, scale, win, sh)
            _check("attn_bwd_ex", st)
        elif Hkv == H:
            st = lib.attn_bwd(*ptrs, B, H, T, D, scale, sh)
            _check("attn_bwd", st)
        else:
            st = lib.attn_bwd_gqa(*ptrs, B, H, Hkv, T, D, scale, sh)
            _check("attn_bwd_gqa", st)
    return dq, dk, dv


def attn_bwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor,
                     dO: torch.Tensor, scale: Optional[float] = None, dq: Optional[torch.Tensor] = None,
                     dk: Optional[torch.Tensor] = None, dv: Optional[torch.Tensor] = None,
                     stream: Optional[torch.cuda.Stream] = None):
    """Backward using the library's built-in scratch array instead of a caller workspace (for callers that
    cannot allocate device memory; sizes up to B*H*roundup(T,128) <= 64512). Returns (dq, dk, dv)."""
    lib = load_library()
    _require_cuda("q", q)
    dq, dk, dv, _ = _bwd_tensors(q, k, v, o, lse, dO, dq, dk, dv, same_heads=True)
    B, T, H, D = q.shape
    scale = default_scale(D) if scale is None else float(scale)
    with torch.cuda.device(q.device):
        st = lib.attn_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                  dO.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, T, D, scale,
                                  _stream_handle(stream, q.device))
    _check("attn_bwd_noalloc", st)
    return dq, dk, dv


def attn_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, cache_seqlens: torch.Tensor,
                scale: Optional[float] = None, o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None,
                window: Optional[int] = None):
    """Attention of Tq new queries against a key/value cache (the inference engine's cached decode).
    q: bf16 [B, Tq, H, D]; k_cache, v_cache: bf16 [B, Tk, H_kv, D]; cache_seqlens: int32 [B] on the device, the
    valid keys of each sequence (new tokens included). Query i, at position p = L - Tq + i, sees keys 0 .. p, or
    with a sliding window keys p - window .. p. Returns (o [B, Tq, H, D], lse [B, H, Tq])."""
    lib = load_library()
    _require_cuda("q", q)
    _check_qkv("q", q)
    dev = q.device
    _check_qkv("k_cache", k_cache, device=dev)
    B, Tq, H, D = q.shape
    Tk, Hkv = k_cache.shape[1], k_cache.shape[2]
    if k_cache.shape[0] != B or k_cache.shape[3] != D:
        raise ValueError(f"k_cache has shape {tuple(k_cache.shape)}; expected [{B}, Tk, H_kv, {D}]")
    _check_qkv("v_cache", v_cache, k_cache.shape, dev)
    if (not isinstance(cache_seqlens, torch.Tensor) or cache_seqlens.dtype != torch.int32 or
            tuple(cache_seqlens.shape) != (B,) or cache_seqlens.device != dev or not cache_seqlens.is_contiguous()):
        raise ValueError("cache_seqlens must be a contiguous int32 [B] tensor on q's device")
    o = torch.empty_like(q) if o is None else o
    _check_qkv("o", o, q.shape, dev)
    if lse is None:
        lse = torch.empty((B, H, Tq), dtype=torch.float32, device=dev)
    _check_f32("lse", lse, (B, H, Tq), dev)
    need = int(lib.attn_decode_workspace_bytes(B, H, Hkv, Tq, Tk, D))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    elif workspace.device != dev:
        raise ValueError(f"workspace is on {workspace.device}; every tensor of one call must be on {dev}")
    scale = default_scale(D) if scale is None else float(scale)
    win = _window_arg(window)
    with torch.cuda.device(dev):
        st = lib.attn_decode_ex(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), cache_seqlens.data_ptr(),
                                o.data_ptr(), lse.data_ptr(), workspace.data_ptr(),
                                workspace.numel() * workspace.element_size(), B, H, Hkv, Tq, Tk, D, scale, win,
                                _stream_handle(stream, dev))
    _check("attn_decode_ex", st)
    return o, lse


ROPE_PAIRINGS = {"interleaved": 0, "half": 1}


def _rope_args(q: torch.Tensor, k: torch.Tensor, pos_offsets: Optional[torch.Tensor], pairing: str):
    _require_cuda("q", q)
    _check_qkv("q", q)
    _check_qkv("k", k)
    B, T, H, D = q.shape
    if (k.shape[0], k.shape[1], k.shape[3]) != (B, T, D) or k.device != q.device:
        raise ValueError(f"k has shape {tuple(k.shape)}; expected [{B}, {T}, H_kv, {D}] on q's device")
    if pairing not in ROPE_PAIRINGS:
        raise ValueError(f"pairing must be one of {sorted(ROPE_PAIRINGS)}, got {pairing!r}")
    ptr = None
    if pos_offsets is not None:
        if (pos_offsets.dtype != torch.int32 or tuple(pos_offsets.shape) != (B,) or
                pos_offsets.device != q.device or not pos_offsets.is_contiguous()):
            raise ValueError("pos_offsets must be a contiguous int32 [B] tensor on q's device")
        ptr = pos_offsets.data_ptr()
    return B, T, H, k.shape[2], D, ptr, ROPE_PAIRINGS[pairing]


def qk_norm_rope(q: torch.Tensor, k: torch.Tensor, rope_base: float = 10000.0, eps: float = 1e-6,
                 pos_offsets: Optional[torch.Tensor] = None, pairing: str = "interleaved", inplace: bool = False,
                 stream: Optional[torch.cuda.Stream] = None):
    """RMS-normalise each head vector of q [B, T, H, D] and k [B, T, H_kv, D], then rotate its pairs by
    position (rotary embedding). Row t of sequence b sits at position pos_offsets[b] + t (int32 [B] on the
    device; None = t). Returns (q_out, k_out), new tensors unless inplace."""
    lib = load_library()
    B, T, H, Hkv, D, offs, pr = _rope_args(q, k, pos_offsets, pairing)
    q_out, k_out = (q, k) if inplace else (torch.empty_like(q), torch.empty_like(k))
    with torch.cuda.device(q.device):
        st = lib.attn_qk_norm_rope(q.data_ptr(), k.data_ptr(), q_out.data_ptr(), k_out.data_ptr(), offs, B, T, H,
                                   Hkv, D, float(rope_base), float(eps), pr, _stream_handle(stream, q.device))
    _check("attn_qk_norm_rope", st)
    return q_out, k_out


def qk_norm_rope_bwd(q: torch.Tensor, k: torch.Tensor, dq_out: torch.Tensor, dk_out: torch.Tensor,
                     rope_base: float = 10000.0, eps: float = 1e-6, pos_offsets: Optional[torch.Tensor] = None,
                     pairing: str = "interleaved", inplace: bool = False, stream: Optional[torch.cuda.Stream] = None):
    """Gradients of q, k (the prologue's inputs) from the gradients dq_out, dk_out of its outputs. With
    inplace the results overwrite dq_out, dk_out."""
    lib = load_library()
    B, T, H, Hkv, D, offs, pr = _rope_args(q, k, pos_offsets, pairing)
    _check_qkv("dq_out", dq_out, q.shape, q.device)
    _check_qkv("dk_out", dk_out, k.shape, q.device)
    dq, dk = (dq_out, dk_out) if inplace else (torch.empty_like(q), torch.empty_like(k))
    with torch.cuda.device(q.device):
        st = lib.attn_qk_norm_rope_bwd(q.data_ptr(), k.data_ptr(), dq_out.data_ptr(), dk_out.data_ptr(),
                                       dq.data_ptr(), dk.data_ptr(), offs, B, T, H, Hkv, D, float(rope_base),
                                       float(eps), pr, _stream_handle(stream, q.device))
    _check("attn_qk_norm_rope_bwd", st)
    return dq, dk


class QKNormRopeFunction(torch.autograd.Function):
    """autograd wrapper of the prologue: forward saves the raw q, k; backward calls qk_norm_rope_bwd."""

    @staticmethod
    def forward(ctx, q, k, rope_base, eps, pos_offsets, pairing):
        q_out, k_out = qk_norm_rope(q, k, rope_base, eps, pos_offsets, pairing)
        ctx.save_for_backward(q, k, pos_offsets)
        ctx.args = (rope_base, eps, pairing)
        return q_out, k_out

    @staticmethod
    def backward(ctx, dq_out, dk_out):
        q, k, pos_offsets = ctx.saved_tensors
        rope_base, eps, pairing = ctx.args
        # out of place: autograd does not promise that the incoming gradient tensors are this function's to change
        dq, dk = qk_norm_rope_bwd(q, k, dq_out.contiguous(), dk_out.contiguous(), rope_base, eps, pos_offsets,
                                  pairing)
        return dq, dk, None, None, None, None


def qk_norm_rope_attention(q, k, v, scale: Optional[float] = None, window: Optional[int] = None,
                           rope_base: float = 10000.0, eps: float = 1e-6, pairing: str = "interleaved"):
    """Differentiable prologue + causal attention: QK normalisation and rotary embedding of q and k, then
    causal_attention. Two launches forward (prologue, attention), the attention backward plus one launch back."""
    qr, kr = QKNormRopeFunction.apply(q, k, rope_base, eps, None, pairing)
    return causal_attention(qr, kr, v, scale, window)


def get_device_error() -> int:
    """The library's device-side error word (0 = no kernel gave up on a bounded wait and, in the debug build, no
    address check failed). Synchronises."""
    word = ctypes.c_uint32(0)
    st = load_library().attn_get_device_error(ctypes.byref(word))
    if st not in (0, 5, 7):
        _check("attn_get_device_error", st)
    return int(word.value)


def clear_device_error():
    _check("attn_clear_device_error", load_library().attn_clear_device_error())


def set_wait_limit_ns(limit_ns: int):
    _check("attn_set_wait_limit_ns", load_library().attn_set_wait_limit_ns(int(limit_ns)))


def selftest_wait_timeout(limit_ns: int, stream: Optional[torch.cuda.Stream] = None):
    dev = torch.device("cuda", torch.cuda.current_device())
    _check("attn_selftest_wait_timeout",
           load_library().attn_selftest_wait_timeout(int(limit_ns), _stream_handle(stream, dev)))


class CausalAttentionFunction(torch.autograd.Function):
    """autograd wrapper: forward saves (q, k, v, o, lse); backward calls attn_bwd."""

    @staticmethod
    def forward(ctx, q, k, v, scale, window=None):
        o, lse = attn_fwd(q, k, v, scale, window=window)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.scale, ctx.window = scale, window
        return o

    @staticmethod
    def backward(ctx, dO):
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = attn_bwd(q, k, v, o, lse, dO.contiguous(), ctx.scale, window=ctx.window)
        return dq, dk, dv, None, None


def causal_attention(q, k, v, scale: Optional[float] = None, window: Optional[int] = None):
    """Differentiable causal attention on bf16 [B, T, H, D] tensors (the flash_attn_func(causal=True,
    window_size=(window, 0)) call); k, v may have fewer heads dividing H (grouped-query attention)."""
    return CausalAttentionFunction.apply(q, k, v, default_scale(q.shape[-1]) if scale is None else scale, window)


__all__ = ["attn_fwd", "attn_bwd", "attn_decode", "attn_bwd_workspace_bytes", "causal_attention", "CausalAttentionFunction",
           "qk_norm_rope", "qk_norm_rope_bwd", "QKNormRopeFunction", "qk_norm_rope_attention",
           "get_device_error", "clear_device_error", "set_wait_limit_ns", "selftest_wait_timeout", "AttnError",
           "load_library", "LIB_PATH", "SIGNATURES"]
