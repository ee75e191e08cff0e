"""Seeded synthetic inputs: determinism, shapes, the recipes of each workload, and the FLOP convention."""
import math

import torch

from workloads import HEADLINE, WORKLOADS, Workload, key_bias_vector, make_inputs, sample_slices


def test_depth_dial_shapes():
    # width = 64 * depth and head_dim 128, so H = depth / 2 (d20: 1280 channels, 10 heads of 128)
    for depth in (12, 20, 24, 26):
        w = WORKLOADS[f"d{depth}"]
        assert w.D == 128 and w.H * w.D == 64 * depth and w.T == 2048
    assert WORKLOADS["d20"].B == 32 and WORKLOADS["d24"].B == 16 and WORKLOADS["d26"].B == 16
    assert HEADLINE == "d20"
    for T in (512, 1024, 2048, 4096):
        w = WORKLOADS[f"d26_T{T}"]
        assert w.B * w.T == 32768 and w.H == 13


def test_inputs_are_deterministic_bf16_and_shaped():
    w = Workload("t", B=2, H=3, T=17, seed=5)
    a = make_inputs(w)
    b = make_inputs(w)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and tuple(x.shape) == (2, 17, 3, 128)
        assert torch.equal(x, y)
    c = make_inputs(w.with_shape(seed=6))
    assert not torch.equal(a[0], c[0])


def test_prescale_is_exact_and_bias_is_shared():
    base = Workload("b", B=1, H=2, T=33, seed=3)
    q0, k0, v0, _ = make_inputs(base)
    q1, k1, v1, _ = make_inputs(base.with_shape(qk_prescale=0.5))
    # multiplying by 0.5 is exact in binary before and after the bf16 rounding
    assert torch.equal(q1.float(), q0.float() * 0.5) and torch.equal(k1.float(), k0.float() * 0.5)
    assert torch.equal(v1, v0)
    wb = base.with_shape(key_bias=True)
    _, kb, _, _ = make_inputs(wb)
    bias = key_bias_vector(wb)
    g = torch.Generator().manual_seed(3)
    draws = [torch.randn((1, 33, 2, 128), generator=g) for _ in range(4)]
    assert torch.equal(kb, (draws[1] + bias).to(torch.bfloat16))


def test_flop_convention():
    w = WORKLOADS["d20"]
    assert w.fwd_flops == 2 * 32 * 10 * 2048 ** 2 * 128
    assert math.isclose(w.fwd_flops + w.bwd_flops, 1.2026e12, rel_tol=1e-4)
    assert math.isclose(w.scale, 1 / math.sqrt(128))


def test_sample_slices_include_corners_and_are_unique():
    w = WORKLOADS["d24"]
    s = sample_slices(w, k=5)
    assert s[0] == (0, 0) and s[1] == (w.B - 1, w.H - 1)
    assert len(set(s)) == len(s) == 5
    assert all(0 <= b < w.B and 0 <= h < w.H for b, h in s)
