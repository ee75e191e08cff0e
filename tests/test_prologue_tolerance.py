"""The prologue's parity bounds are neither too tight nor too loose (CPU).

A float32 model of the kernels' arithmetic (sum of squares, reciprocal square root, the angle as a double
product reduced exactly to [-1, 1] half-turns and then a single-precision sin/cos of pi times it, the rotation,
bf16 rounding of the output) must pass the bounds of tests/prologue_checks.py on every parity case: the bounds
leave room for that arithmetic. A model with one plausible precision mistake, the whole angle computed in
float32 (position times frequency rounded to single precision before the sin/cos), must fail them on the
large position offsets of rope_tiny: the bounds are tight enough to see it. The model is a restatement of the
kernels' arithmetic in numpy for this check only; it is not the oracle and not the CUDA path.
"""
import dataclasses

import numpy as np
import pytest
import torch

from oracle import attn_ref
from prologue_checks import check_bwd, check_fwd, oracle_kwargs
from workloads import PROLOGUE_WORKLOADS, make_prologue_inputs

F32 = np.float32


def bf16_round(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=F32)).to(torch.bfloat16).double().numpy()


def kernel_model(x, dy, w, offsets, float32_angle=False):
    """(y, dx) as the kernels compute them, in float32, rounded to bf16."""
    x, dy = x.float().numpy(), dy.float().numpy()
    B, T, H, D = x.shape
    off = np.zeros(B) if offsets is None else np.asarray(offsets, dtype=np.float64)
    pos = off[:, None] + np.arange(T)
    pair = np.arange(D) // 2 if w.pairing == "interleaved" else np.arange(D) % (D // 2)
    half_turns = w.rope_base ** (-pair / (D / 2)) / np.pi                  # frequency in half-turns, double
    if float32_angle:
        u = (pos.astype(F32)[:, :, None] * half_turns.astype(F32)[None, None, :]).astype(np.float64)
    else:
        u = pos[:, :, None] * half_turns[None, None, :]
        u = u - 2.0 * np.rint(0.5 * u)                                       # exact reduction
    u = u.astype(F32).astype(np.float64)
    cs = np.cos(np.pi * u).astype(F32)[:, :, None, :]
    sn = np.sin(np.pi * u).astype(F32)[:, :, None, :]
    idx = np.arange(D)
    if w.pairing == "interleaved":
        sign, partner = np.where(idx % 2 == 1, 1, -1).astype(F32), idx ^ 1
    else:
        sign, partner = np.where(idx >= D // 2, 1, -1).astype(F32), (idx + D // 2) % D
    r = (F32(1) / np.sqrt((x * x).sum(-1, keepdims=True, dtype=F32) / F32(D) + F32(w.eps))).astype(F32)
    y = (x * r) * cs + sign * (x[..., partner] * r) * sn
    g = dy * cs - sign * dy[..., partner] * sn
    dot = (g * (x * r)).sum(-1, keepdims=True, dtype=F32) / F32(D)
    dx = r * (g - (x * r) * dot)
    return bf16_round(y), bf16_round(dx)


CASES = [{}, {"pairing": "half"}, {"eps": 0.0, "rope_base": 500.0}, {"max_offset": 0, "H": 3, "Hkv": 1},
         {"B": 1, "T": 1, "H": 1, "Hkv": 1}, {"B": 3, "T": 300, "H": 2, "Hkv": 2, "pairing": "half", "max_offset": 0}]


@pytest.mark.parametrize("changes", CASES)
def test_kernel_arithmetic_fits_the_bounds(changes):
    w = dataclasses.replace(PROLOGUE_WORKLOADS["rope_tiny"], **changes)
    q, k, gq, gk, offs = make_prologue_inputs(w)
    offsets = None if offs is None else offs.numpy()
    kw = oracle_kwargs(w, offsets)
    for name, x, dy in (("q", q, gq), ("k", k, gk)):
        y, dx = kernel_model(x, dy, w, offsets)
        check_fwd(y, attn_ref.qk_norm_rope(x, **kw), f"{changes} {name}")
        check_bwd(dx, attn_ref.qk_norm_rope_backward(x, dy, **kw), x, dy, w.eps, f"{changes} {name} backward")


def test_bounds_catch_a_single_precision_angle():
    w = PROLOGUE_WORKLOADS["rope_tiny"]  # offsets up to 1e5: an angle rounded to float32 is off by ~1e-3 rad
    q, k, gq, gk, offs = make_prologue_inputs(w)
    kw = oracle_kwargs(w, offs.numpy())
    y, _ = kernel_model(q, gq, w, offs.numpy(), float32_angle=True)
    with pytest.raises(AssertionError):
        check_fwd(y, attn_ref.qk_norm_rope(q, **kw), "float32 angle")
