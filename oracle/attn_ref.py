"""Float64 CPU oracle for bf16 causal multi-head self-attention, forward and backward.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import this module. It shares no code with the CUDA path and never calls it.

What it computes. The pages call the attention as ``flash_attn_func(q, k, v, causal=True, window_size=...)`` on
[B, T, H, D] tensors (apidog "Train your own ChatGPT", section 5 "Flash Attention integration", and section 1
"GPT model" for the [B, T, n_head, head_dim] view); the model trains through it, so a backward exists. The pages
print neither the formula nor the backward, so this file writes out the textbook definition of scaled
dot-product attention under a causal mask, the one the pages' SDPA fallback computes (same section 5):

  per (b, h), with s the softmax scale and i, j query/key positions,
    S[i, j]  = s * sum_d Q[i, d] K[j, d]     for j <= i,   -inf for j > i   (top-left aligned, T_q = T_k)
    m_i      = max_j S[i, j],   l_i = sum_j exp(S[i, j] - m_i)
    P[i, j]  = exp(S[i, j] - m_i) / l_i
    O        = P V
    LSE_i    = m_i + ln l_i                     (natural log of the scaled, masked logits)
  and, for an upstream gradient dO of a loss L = sum(dO * O):
    dV       = P^T dO
    dP       = dO V^T
    Delta_i  = sum_d dO[i, d] O[i, d]          (= sum_j P[i, j] dP[i, j])
    dS       = P * (dP - Delta)                 (zero where masked, because P is)
    dQ       = s dS K,      dK = s dS^T Q

Everything is dense over the full T x T matrix of each (b, h) and masked afterwards: no blocking, no online
softmax, no reordering. A blockwise online-softmax kernel reaches the same values in exact arithmetic.

Readings where the pages are silent: scale = 1/sqrt(D) passed explicitly; mask aligned top-left; LSE in
natural log over the scaled logits; inputs are bf16 values upcast exactly to float64 with no intermediate
rounding here (the GPU rounds P and dS to bf16 before its matrix products; the parity tolerances absorb that).

Pins (tests/test_oracle.py): softmax rows sum to one; causality under perturbation of later positions; T = 1;
Q = 0 closed form (prefix mean, LSE = ln(t + 1)); equal keys; shift invariance of the keys; agreement with
torch's float64 ``scaled_dot_product_attention`` and its autograd; central finite differences; the Delta
identity; a hand-derived worked example under tests/golden/.

Also here: grouped-query heads and the sliding window (``kv_group``, ``causal_mask``), cached decode
(``decode_forward``), and the QK-normalisation + rotary-embedding prologue with its backward
(``qk_norm_rope``, ``qk_norm_rope_backward``; RMS normalisation and the RoFormer rotation, readings stated in
their docstrings). The prologue is pinned by the complex-exponential form of the rotation, relative-position
invariance, a closed-form eps case, the agreement of the two pairings under a permutation, and central finite
differences of the backward.
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np


def _as_f64(x) -> np.ndarray:
    """Upcast an array-like (numpy, or a CPU torch tensor of any float dtype) to float64 numpy, exactly."""
    if hasattr(x, "detach"):
        import torch  # local: the oracle itself is numpy; torch only as an input container
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def causal_mask(T: int, window: Optional[int] = None) -> np.ndarray:
    """Boolean [T, T] matrix, True where key j may be seen by query i: j <= i, and with a sliding window also
    j >= i - window, so a query sees itself and the `window` keys before it. The pages pass
    ``window_size=window_size`` to flash_attn_func and alternate short- and long-window layers ("SSSL") (apidog
    "Train your own ChatGPT", section 1 "GPT model" and section 5 "Flash Attention integration"); reading:
    flash_attn's left window, causal on the right; None is no window."""
    m = np.tril(np.ones((T, T), dtype=bool))
    if window is not None:
        if window < 0:
            raise ValueError("window must be >= 0 (or None for no window)")
        m &= np.triu(np.ones((T, T), dtype=bool), -window)  # j - i >= -window
    return m


def head_forward(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float, window: Optional[int] = None):
    """Forward of one (b, h) slice: q, k, v are [T, D] float64. Returns (O [T, D], LSE [T], P [T, T])."""
    T = q.shape[0]
    S = scale * (q @ k.T)
    S = np.where(causal_mask(T, window), S, -np.inf)
    m = S.max(axis=1, keepdims=True)           # finite: the diagonal is always visible
    E = np.exp(S - m)                          # exp(-inf) = 0 on masked entries
    l = E.sum(axis=1, keepdims=True)
    P = E / l
    O = P @ v
    lse = (m + np.log(l))[:, 0]
    return O, lse, P


def head_backward(q, k, v, do, scale: float, o=None, window: Optional[int] = None):
    """Backward of one (b, h) slice from the definition. Returns (dQ, dK, dV, Delta).

    ``o`` is the forward output used for Delta; by default the exact float64 output of ``head_forward``.
    """
    O, _, P = head_forward(q, k, v, scale, window)
    if o is None:
        o = O
    dV = P.T @ do
    dP = do @ v.T
    delta = (do * o).sum(axis=1)
    dS = P * (dP - delta[:, None])
    dQ = scale * (dS @ k)
    dK = scale * (dS.T @ q)
    return dQ, dK, dV, delta


def kv_group(H: int, Hkv: int) -> int:
    """Query heads per key/value head. Grouped-query attention (apidog "Train your own ChatGPT", section 1 "GPT
    model": fewer key/value heads than query heads, the value tensor viewed with n_kv_head heads) gives query
    head h the key/value head h // (H // H_kv): consecutive query heads share one (the pages do not print the
    mapping; this is the plainest reading, and H_kv = H is plain multi-head attention)."""
    if Hkv < 1 or H % Hkv:
        raise ValueError(f"H = {H} query heads cannot be grouped over H_kv = {Hkv} key/value heads")
    return H // Hkv


def attention_forward(q, k, v, scale: float, window: Optional[int] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Full forward over q [B, T, H, D] and k, v [B, T, H_kv, D] (H_kv divides H; H_kv = H is multi-head
    attention). Returns O [B, T, H, D] and LSE [B, H, T], both float64."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, T, H, D = q.shape
    G = kv_group(H, k.shape[2])
    O = np.empty((B, T, H, D))
    LSE = np.empty((B, H, T))
    for b in range(B):
        for h in range(H):
            o_bh, lse_bh, _ = head_forward(q[b, :, h], k[b, :, h // G], v[b, :, h // G], scale, window)
            O[b, :, h] = o_bh
            LSE[b, h] = lse_bh
    return O, LSE


def attention_backward(q, k, v, do, scale: float, o=None, window: Optional[int] = None):
    """Full backward over q, dO [B, T, H, D] and k, v [B, T, H_kv, D]. Returns dQ [B, T, H, D], dK, dV
    [B, T, H_kv, D] and Delta [B, H, T]. A key/value head feeds every query head of its group, so its gradient
    is the sum of the per-head gradients over the group (the chain rule over the shared input)."""
    q, k, v, do = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(do)
    o = None if o is None else _as_f64(o)
    B, T, H, D = q.shape
    G = kv_group(H, k.shape[2])
    dQ, dK, dV = np.empty_like(q), np.zeros_like(k), np.zeros_like(v)
    delta = np.empty((B, H, T))
    for b in range(B):
        for h in range(H):
            o_bh = None if o is None else o[b, :, h]
            gq, gk, gv, dl = head_backward(q[b, :, h], k[b, :, h // G], v[b, :, h // G], do[b, :, h], scale, o_bh,
                                           window)
            dQ[b, :, h] = gq
            dK[b, :, h // G] += gk
            dV[b, :, h // G] += gv
            delta[b, h] = dl
    return dQ, dK, dV, delta


def slice_forward_backward(q, k, v, do, b: int, h: int, scale: float, window: Optional[int] = None):
    """Forward and backward of the single (b, h) query-head slice (slices are independent). q, dO are
    [B, T, H, D], k, v [B, T, H_kv, D]; the slice reads key/value head h // (H // H_kv).

    Returns a dict of float64 arrays: o [T, D], lse [T], dq, dk, dv [T, D], delta [T]; dk, dv are this query
    head's contributions (a key/value head's gradient is their sum over its group).
    """
    hk = h // kv_group(q.shape[2], k.shape[2])
    qs, ks, vs = _as_f64(q[b, :, h]), _as_f64(k[b, :, hk]), _as_f64(v[b, :, hk])
    o, lse, _ = head_forward(qs, ks, vs, scale, window)
    out = {"o": o, "lse": lse}
    if do is not None:
        dos = _as_f64(do[b, :, h])
        dq, dk, dv, delta = head_backward(qs, ks, vs, dos, scale, window=window)
        out.update(dq=dq, dk=dk, dv=dv, delta=delta)
    return out


def decode_forward(q, k_cache, v_cache, cache_seqlens, scale: float,
                   window: Optional[int] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Attention of a few new queries against a key/value cache (the inference engine's
    flash_attn_with_kvcache over a prefilled cache: apidog "Train your own ChatGPT", section 6 "Inference
    engine").

    q: [B, Tq, H, D]; k_cache, v_cache: [B, Tk, H_kv, D] (H_kv divides H, grouped as in ``attention_forward``);
    cache_seqlens: [B] integers, the number of valid cached keys of each sequence, the Tq new tokens' keys
    included (the caller has written them). Reading (the pages give no more): query i of sequence b sits at
    position p = L_b - Tq + i and sees keys 0 .. p (causal, aligned to the end of the cache); with a sliding
    window (the model's short-window layers, section 1 "GPT model", decoded through the same call) only keys
    p - window .. p, the band of ``causal_mask``. A query that sees no key (p < 0) returns O = 0 and
    LSE = -inf. Returns O [B, Tq, H, D], LSE [B, H, Tq].
    """
    q, kc, vc = _as_f64(q), _as_f64(k_cache), _as_f64(v_cache)
    B, Tq, H, D = q.shape
    G = kv_group(H, kc.shape[2])
    lens = np.asarray(cache_seqlens, dtype=np.int64).reshape(-1)
    if lens.shape[0] != B or (lens < 0).any() or (lens > kc.shape[1]).any():
        raise ValueError("cache_seqlens must hold B lengths in [0, Tk]")
    if window is not None and window < 0:
        raise ValueError("window must be >= 0 or None")
    O = np.zeros((B, Tq, H, D))
    LSE = np.full((B, H, Tq), -np.inf)
    for b in range(B):
        L = int(lens[b])
        for h in range(H):
            k, v = kc[b, :L, h // G], vc[b, :L, h // G]
            for i in range(Tq):
                last = L - Tq + i                      # last visible key: the query's own position
                if last < 0:
                    continue
                first = 0 if window is None else max(0, last - window)
                s = scale * (k[first: last + 1] @ q[b, i, h])
                m = s.max()
                e = np.exp(s - m)
                O[b, i, h] = (e @ v[first: last + 1]) / e.sum()
                LSE[b, h, i] = m + np.log(e.sum())
    return O, LSE


def _rope_angles(B: int, T: int, D: int, base: float, offsets) -> np.ndarray:
    """Rotation angles [B, T, D/2]: position p = offsets[b] + t (offsets a scalar or a length-B array) times
    the frequency base^(-2i/D) of pair i (RoFormer, Su et al. 2021, section 3.4.2)."""
    off = np.broadcast_to(np.asarray(offsets, dtype=np.float64), (B,))
    pos = off[:, None] + np.arange(T, dtype=np.float64)[None, :]          # [B, T]
    inv_freq = float(base) ** (-2.0 * np.arange(D // 2) / D)               # [D/2]
    return pos[:, :, None] * inv_freq[None, None, :]


def _pairs(y: np.ndarray, pairing: str):
    """The (first, second) members of each rotated pair: interleaved (2i, 2i+1), or half (i, i + D/2)."""
    D = y.shape[-1]
    if pairing == "interleaved":
        return y[..., 0::2], y[..., 1::2]
    if pairing == "half":
        return y[..., : D // 2], y[..., D // 2:]
    raise ValueError(f"pairing must be 'interleaved' or 'half', got {pairing!r}")


def _unpairs(a: np.ndarray, b: np.ndarray, pairing: str) -> np.ndarray:
    out = np.empty(a.shape[:-1] + (2 * a.shape[-1],))
    if pairing == "interleaved":
        out[..., 0::2], out[..., 1::2] = a, b
    else:
        out = np.concatenate([a, b], axis=-1)
    return out


def qk_norm_rope(x, base: float = 10000.0, eps: float = 1e-6, offsets=0, pairing: str = "interleaved") -> np.ndarray:
    """The steps the model applies to q and k before attention (apidog "Train your own ChatGPT", section 1 "GPT
    model", architecture features: rotary embeddings for relative positions without learned position
    embeddings, and QK normalisation for stability; the pages give neither formula). Readings:
      * QK normalisation: RMS normalisation of each head vector over D without a learnable weight,
        y = x / sqrt(mean(x^2) + eps);
      * rotary embedding (RoFormer, Su et al. 2021): each pair (first, second) of y at position p is turned by
        the angle p * base^(-2i/D), first' = first cos - second sin, second' = first sin + second cos. Pair i
        is (2i, 2i+1) ("interleaved", the paper's form) or (i, i + D/2) ("half");
      * positions: row t of sequence b sits at offsets[b] + t (0 for a training batch; the cache length
        before the new tokens for decode).
    Rotation keeps the RMS, so the two steps commute.

    x: [B, T, H, D] (q, or k with its own head count). Returns float64 [B, T, H, D].
    """
    x = _as_f64(x)
    B, T, H, D = x.shape
    y = x / np.sqrt((x * x).mean(axis=-1, keepdims=True) + eps)
    ang = _rope_angles(B, T, D, base, offsets)[:, :, None, :]              # [B, T, 1, D/2]
    c, s = np.cos(ang), np.sin(ang)
    a, b = _pairs(y, pairing)
    return _unpairs(a * c - b * s, a * s + b * c, pairing)


def qk_norm_rope_backward(x, dy, base: float = 10000.0, eps: float = 1e-6, offsets=0,
                          pairing: str = "interleaved") -> np.ndarray:
    """Gradient of sum(dy * qk_norm_rope(x)) with respect to x, by the chain rule through the two steps:
      * rotation: the transpose turns each pair back by the same angle, g = R(-angle) dy;
      * RMS normalisation y = x r, r = (mean(x^2) + eps)^(-1/2): dx = r (g - y mean(g y)).
    Returns float64 [B, T, H, D].
    """
    x, dy = _as_f64(x), _as_f64(dy)
    B, T, H, D = x.shape
    r = 1.0 / np.sqrt((x * x).mean(axis=-1, keepdims=True) + eps)
    y = x * r
    ang = _rope_angles(B, T, D, base, offsets)[:, :, None, :]
    c, s = np.cos(ang), np.sin(ang)
    a, b = _pairs(dy, pairing)
    g = _unpairs(a * c + b * s, -a * s + b * c, pairing)
    return r * (g - y * (g * y).mean(axis=-1, keepdims=True))
