"""The forward kernel's software exp2 (attn_fwd.cuh, exp2_poly): its algorithm, emulated step by step in
float32, stays within the fitted relative-error bound over the whole softmax argument range, and the
kernel's constants are the ones the fitting script produces."""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "causal_self_attention_bf16_b200", "csrc")
sys.path.insert(0, CSRC)
import fit_exp2_poly  # noqa: E402

BOUND = 8e-5  # fitted bound 7.5e-5, plus float32 rounding of the steps


def emulate(x):
    f32 = np.float32
    x = x.astype(f32)
    magic = f32(12582912.0)
    t = (x + magic).astype(f32)
    f = (x - (t - magic).astype(f32)).astype(f32)
    c0, c1, c2, c3 = (np.float64(v) for v in (0.999928073, 0.693260987, 0.242611135, 0.0551716668))
    p = (((c3 * f + c2) * f + c1) * f + c0).astype(f32)
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    r = (bits & 0xFFFFFFFF).astype(np.uint32).view(np.int32).view(f32)
    return np.where(x < f32(-126.0), f32(0.0), r)


def test_relative_error_over_softmax_range():
    x = np.concatenate([np.linspace(-125.0, 8.0, 400001), np.linspace(-1.0, 1.0, 20001)]).astype(np.float32)
    got = emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < BOUND, rel.max()


def test_underflow_and_masked_keys_give_zero():
    with np.errstate(invalid="ignore", over="ignore"):
        got = emulate(np.array([-126.5, -200.0, -1e30, -np.inf], dtype=np.float32))
    assert np.all(got == 0.0)
    assert 0 < emulate(np.array([-126.0], dtype=np.float32))[0] < 2e-38


def test_kernel_constants_match_the_fit():
    fitted = fit_exp2_poly.fit()
    src = open(os.path.join(CSRC, "attn_fwd.cuh")).read()
    body = src[src.index("float exp2_poly(float x)"):]
    body = body[:body.index("\n}")]
    consts = [float(v) for v in re.findall(r"(\d+\.\d+)f", body) if v not in ("126.0", "12582912.0", "0.0")]
    c3, c2, c1, c0 = consts
    np.testing.assert_allclose([c0, c1, c2, c3], fitted, rtol=1e-7)
