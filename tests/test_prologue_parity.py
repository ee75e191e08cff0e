"""Parity of the QK-normalisation + rotary-embedding prologue (through the C ABI) with the float64 oracle.

Tolerances, derived from the arithmetic (the pages give none), per element:
  forward : |y - y_ref| <= 2^-8 |y_ref| + 1e-4. The kernel computes in fp32 and rounds y to bf16, half an
            ulp being at most 2^-8 of the value; the fp32 sum of 128 squares, rsqrtf, the angle (reduced
            exactly in double, then sincospif) and the rotation leave under 1e-5 in these units (every row
            has RMS 1 after the normalisation).
  backward: |dx - dx_ref| <= 2^-8 |dx_ref| + 1e-4 r max|dy_row|, with r = (mean(x^2) + eps)^(-1/2) of the row:
            r max|dy| is the scale of dx = r (g - y mean(g y)), and the fp32 error stays below 1e-5 of it.
Small cases compare every element; the full-size workloads compare seeded runs of 16 positions, which the
oracle computes one by one (a run starting at time t0 is the oracle at offset t0).
"""
import dataclasses

import numpy as np
import pytest
import torch

import causal_self_attention_bf16_b200 as attn
from oracle import attn_ref
from prologue_checks import check_bwd, check_fwd, oracle_kwargs
from workloads import PROLOGUE_WORKLOADS, WORKLOADS, make_inputs, make_prologue_inputs

pytestmark = pytest.mark.gpu


def to64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def run_case(w, inplace=False):
    dev = torch.device("cuda")
    q, k, dq_out, dk_out, offs = make_prologue_inputs(w)
    qd, kd, gqd, gkd = (t.to(dev) for t in (q, k, dq_out, dk_out))
    od = None if offs is None else offs.to(dev)
    if inplace:
        q_in, k_in = qd.clone(), kd.clone()
        yq, yk = attn.qk_norm_rope(q_in, k_in, w.rope_base, w.eps, od, w.pairing, inplace=True)
        assert yq.data_ptr() == q_in.data_ptr() and yk.data_ptr() == k_in.data_ptr()
    else:
        yq, yk = attn.qk_norm_rope(qd, kd, w.rope_base, w.eps, od, w.pairing)
    dq, dk = attn.qk_norm_rope_bwd(qd, kd, gqd, gkd, w.rope_base, w.eps, od, w.pairing, inplace=inplace)
    torch.cuda.synchronize()
    offsets = None if offs is None else offs.numpy()
    return (q, k, dq_out, dk_out, offsets), (to64(yq), to64(yk), to64(dq), to64(dk))


CASES = [
    ("rope_tiny", {}),
    ("rope_tiny", {"pairing": "half"}),
    ("rope_tiny", {"eps": 0.0, "rope_base": 500.0}),
    ("rope_tiny", {"max_offset": 0, "H": 3, "Hkv": 1}),         # 4 rows per position: one unrolled group
    ("rope_tiny", {"B": 1, "T": 1, "H": 1, "Hkv": 1}),          # one position, 2 rows
    ("rope_tiny", {"B": 3, "T": 300, "H": 2, "Hkv": 2, "pairing": "half", "max_offset": 0}),
]


@pytest.mark.parametrize("name,changes", CASES)
def test_prologue_matches_oracle(name, changes):
    w = dataclasses.replace(PROLOGUE_WORKLOADS[name], **changes)
    (q, k, gq, gk, offs), (yq, yk, dq, dk) = run_case(w)
    kw = oracle_kwargs(w, offs)
    what = f"{name} {changes}"
    check_fwd(yq, attn_ref.qk_norm_rope(q, **kw), what + " q")
    check_fwd(yk, attn_ref.qk_norm_rope(k, **kw), what + " k")
    check_bwd(dq, attn_ref.qk_norm_rope_backward(q, gq, **kw), q, gq, w.eps, what + " dq")
    check_bwd(dk, attn_ref.qk_norm_rope_backward(k, gk, **kw), k, gk, w.eps, what + " dk")


def test_prologue_in_place_matches_out_of_place():
    w = PROLOGUE_WORKLOADS["rope_tiny"]
    _, a = run_case(w)
    _, b = run_case(w, inplace=True)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_prologue_zero_row_gives_zero():
    """A zero head vector with eps > 0 normalises to zero (and its gradient is r * g, finite)."""
    w = dataclasses.replace(PROLOGUE_WORKLOADS["rope_tiny"], B=1, T=5, H=2, Hkv=1)
    dev = torch.device("cuda")
    q, k, gq, gk, offs = make_prologue_inputs(w)
    q[0, 2, 1] = 0
    yq, _ = attn.qk_norm_rope(q.to(dev), k.to(dev), w.rope_base, w.eps, offs.to(dev), w.pairing)
    dq, _ = attn.qk_norm_rope_bwd(q.to(dev), k.to(dev), gq.to(dev), gk.to(dev), w.rope_base, w.eps, offs.to(dev),
                                  w.pairing)
    torch.cuda.synchronize()
    assert torch.count_nonzero(yq[0, 2, 1]).item() == 0
    kw = oracle_kwargs(w, offs.numpy())
    check_bwd(to64(dq), attn_ref.qk_norm_rope_backward(q, gq, **kw), q, gq, w.eps, "zero row dq")


@pytest.mark.parametrize("name", ["rope_d20", "rope_d20_gqa"])
def test_prologue_full_size_sampled(name):
    """The benchmark's workloads: every row computed on the GPU, seeded runs of 16 positions checked."""
    w = PROLOGUE_WORKLOADS[name]
    (q, k, gq, gk, _), (yq, yk, dq, dk) = run_case(w)
    rng = np.random.default_rng(5)
    runs = [(0, 0), (w.B - 1, w.T - 16)] + [(int(rng.integers(w.B)), int(rng.integers(w.T - 16))) for _ in range(4)]
    for b, t0 in runs:
        sl = (slice(b, b + 1), slice(t0, t0 + 16))
        kw = oracle_kwargs(w, t0)
        what = f"{name} b={b} t0={t0}"
        check_fwd(yq[sl], attn_ref.qk_norm_rope(q[sl], **kw), what + " q")
        check_fwd(yk[sl], attn_ref.qk_norm_rope(k[sl], **kw), what + " k")
        check_bwd(dq[sl], attn_ref.qk_norm_rope_backward(q[sl], gq[sl], **kw), q[sl], gq[sl], w.eps, what + " dq")
        check_bwd(dk[sl], attn_ref.qk_norm_rope_backward(k[sl], gk[sl], **kw), k[sl], gk[sl], w.eps, what + " dk")


@pytest.mark.parametrize("pairing", ["interleaved", "half"])
def test_prologue_then_attention_through_autograd(pairing):
    """qk_norm_rope_attention (prologue, then causal attention) against the oracle chain: the prologue, the
    attention forward and backward, and the prologue backward, all in float64. The attention bounds apply
    (the GPU also rounds the normalised q, k to bf16 before attention)."""
    w = WORKLOADS["tiny_gqa"].with_shape(T=200)
    q, k, v, do = make_inputs(w)
    dev = torch.device("cuda")
    qd, kd, vd = (t.to(dev).requires_grad_(True) for t in (q, k, v))
    o = attn.qk_norm_rope_attention(qd, kd, vd, w.scale, pairing=pairing)
    o.backward(do.to(dev))
    torch.cuda.synchronize()
    kw = dict(pairing=pairing)
    yq, yk = attn_ref.qk_norm_rope(q, **kw), attn_ref.qk_norm_rope(k, **kw)
    O_ref, _ = attn_ref.attention_forward(yq, yk, v, w.scale)
    dYq, dYk, dV_ref, _ = attn_ref.attention_backward(yq, yk, v, do, w.scale)
    dQ_ref = attn_ref.qk_norm_rope_backward(q, dYq, **kw)
    dK_ref = attn_ref.qk_norm_rope_backward(k, dYk, **kw)
    err = np.abs(to64(o) - O_ref).max()
    assert err <= 1e-2 * np.abs(O_ref).max() + 1e-3, f"O max err {err:.3e}"
    for name, g, r in (("dQ", qd.grad, dQ_ref), ("dK", kd.grad, dK_ref), ("dV", vd.grad, dV_ref)):
        rel = np.linalg.norm(to64(g) - r) / np.linalg.norm(r)
        assert rel <= 2e-2, f"{name} relative Frobenius error {rel:.3e}"
