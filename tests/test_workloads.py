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


def test_grouped_query_inputs_and_key_bias_stream():
    """k, v carry H_kv heads; the draw order q, k, v, dO, bias is kept when the key/value heads differ."""
    w = WORKLOADS["tiny_gqa"]
    q, k, v, do = make_inputs(w)
    assert tuple(q.shape) == tuple(do.shape) == (1, 128, 4, 128)
    assert tuple(k.shape) == tuple(v.shape) == (1, 128, 2, 128) and w.kv_heads == 2
    wb = Workload("gb", B=1, H=4, T=9, Hkv=2, seed=4, key_bias=True)
    _, kb, _, _ = make_inputs(wb)
    g = torch.Generator().manual_seed(4)
    q_ = torch.randn((1, 9, 4, 128), generator=g)
    k_ = torch.randn((1, 9, 2, 128), generator=g)
    assert torch.equal(kb, (k_ + key_bias_vector(wb)).to(torch.bfloat16))


def test_window_flops_scale_with_the_pairs_inside_the_band():
    """A window keeps min(i, W) + 1 of query i's causal keys; W >= T - 1 is the plain causal count."""
    full = WORKLOADS["d20"]
    assert full.with_shape(window=full.T - 1).fwd_flops == full.fwd_flops
    w = Workload("w", B=1, H=1, T=10, window=3)
    kept = sum(min(i, 3) + 1 for i in range(10))          # 1 + 2 + 3 + 4 * 7 = 34 of 55 causal pairs
    assert math.isclose(w.fwd_flops, 2 * 10 * 10 * 128 * kept / 55)
    sw = WORKLOADS["d20_sw"]
    assert 0.4 < sw.fwd_flops / full.fwd_flops < 0.45 and math.isclose(sw.bwd_flops, 2.5 * sw.fwd_flops)


def test_decode_inputs_are_seeded_and_ragged():
    from workloads import DECODE_WORKLOADS, make_decode_inputs
    w = DECODE_WORKLOADS["decode_d20_gqa"]
    q, kc, vc, lens = make_decode_inputs(w)
    q2, kc2, vc2, lens2 = make_decode_inputs(w)
    assert torch.equal(lens, lens2) and torch.equal(q, q2) and torch.equal(kc, kc2)
    assert tuple(q.shape) == (64, 1, 10, 128) and tuple(kc.shape) == (64, 2048, 5, 128)
    assert lens.dtype == torch.int32 and int(lens.min()) >= 1 and int(lens.max()) <= 2048
    assert len(set(lens.tolist())) > 40  # a mix of lengths, not one


def test_bench_decode_bytes_count_only_valid_cache_rows():
    import bench
    from workloads import DECODE_WORKLOADS
    w = DECODE_WORKLOADS["decode_tiny"]
    lens = torch.tensor([10, 0, 5], dtype=torch.int32)
    kv = 15 * w.Hkv * w.D * 2 * 2
    assert bench.decode_bytes(w, lens) == kv + 2 * w.B * w.Tq * w.H * w.D * 2 + w.B * w.H * w.Tq * 4
    f, b = bench.flops(WORKLOADS["d20_sw"])
    assert f == WORKLOADS["d20_sw"].fwd_flops and b == WORKLOADS["d20_sw"].bwd_flops


def test_prologue_inputs_and_bytes():
    """Seeded, shaped prologue inputs (offsets only when asked for), and the byte count of one step: the forward
    reads and writes every row of q and k, the backward reads two and writes one."""
    import bench
    from workloads import PROLOGUE_WORKLOADS, make_prologue_inputs
    w = PROLOGUE_WORKLOADS["rope_tiny"]
    a, b = make_prologue_inputs(w), make_prologue_inputs(w)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    q, k, dq, dk, offs = a
    assert tuple(q.shape) == tuple(dq.shape) == (2, 37, 5, 128) and tuple(k.shape) == tuple(dk.shape) == (2, 37, 2, 128)
    assert q.dtype == k.dtype == torch.bfloat16 and offs.dtype == torch.int32 and tuple(offs.shape) == (2,)
    assert int(offs.min()) >= 0 and int(offs.max()) <= w.max_offset
    norms = q.float().pow(2).mean(-1).sqrt().flatten()
    assert norms.max() / norms.min() > 2.0  # rows of different size, so the normalisation matters
    assert make_prologue_inputs(PROLOGUE_WORKLOADS["rope_d20"].__class__("x", B=1, T=3, H=1, Hkv=1))[4] is None
    row = 32 * 2048 * 20 * 128 * 2
    assert bench.prologue_bytes(PROLOGUE_WORKLOADS["rope_d20"]) == (2 * row, 3 * row)


def test_clock_summary_parses_nvidia_smi_rows():
    """The clocks object of the bench line: median SM clock under load, max clock and power, and throttle
    reasons seen Active in any sample; unparsable rows are skipped."""
    import bench
    text = "\n".join([
        "0, 1965, 1965, 700.5, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1897, 1965, 998.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1830, 1965, 1001.2, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, [N/A], 1965, 10.0, 0x0, Not Active, Active, Not Active, Not Active",   # skipped entirely
        "0, 1965, 19",                                                               # cut off
    ])
    c = bench.summarize_clocks(text)
    assert c["samples"] == 3 and c["sm_mhz"] == 1897.0 and c["sm_max_mhz"] == 1965.0
    assert c["power_w_max"] == 1001.2 and c["reasons"] == ["sw_power_cap"]
    empty = bench.summarize_clocks("")
    assert empty["samples"] == 0 and empty["sm_mhz"] is None and empty["reasons"] == []
