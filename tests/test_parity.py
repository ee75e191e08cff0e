"""Parity of the CUDA path (through the C ABI) with the float64 oracle.

Tolerances (stated for the rebuilt path; the pages give none):
  O      : max|err| <= 1e-2 * max|ref| + 1e-3
  dQ/dK/dV: ||gpu - ref||_F / ||ref||_F <= 2e-2
  LSE    : max|err| <= 1e-3 * max(1, |ref|)
The GPU rounds inputs to bf16 (the oracle sees the same bf16 values), rounds P and dS to bf16 before its
matrix products and rounds outputs to bf16; these bounds leave room for that and nothing else.

Small cases compare every element; the full-size workloads (exactly the shapes and the launch the benchmark
times) compare seeded (b, h) slices, which are independent problems the oracle computes one by one.
"""
import math

import numpy as np
import pytest
import torch

import causal_self_attention_bf16_b200 as attn
from oracle import attn_ref
from workloads import WORKLOADS, Workload, make_inputs, sample_slices

pytestmark = pytest.mark.gpu

O_REL, O_ABS = 1e-2, 1e-3
GRAD_FRO = 2e-2
LSE_TOL = 1e-3


def check_o(o_gpu, o_ref, what=""):
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    err = np.abs(o_gpu - o_ref).max()
    bound = O_REL * np.abs(o_ref).max() + O_ABS
    assert err <= bound, f"{what} O: max err {err:.3e} > {bound:.3e}"


def check_lse(l_gpu, l_ref, what=""):
    err = np.abs(np.asarray(l_gpu, dtype=np.float64) - l_ref)
    assert np.all(err <= LSE_TOL * np.maximum(1.0, np.abs(l_ref))), f"{what} LSE: max err {err.max():.3e}"


def check_grad(g_gpu, g_ref, name, what=""):
    g_gpu = np.asarray(g_gpu, dtype=np.float64)
    assert np.all(np.isfinite(g_gpu)), f"{what} {name}: non-finite values"
    if np.linalg.norm(g_ref) < 1e-9:
        # The exact gradient is zero (T = 1 gives dQ = dK = 0); a relative error is undefined, so bound the
        # fp32 rounding of dP - Delta that is all the kernels can leave.
        assert np.abs(g_gpu).max() < 1e-2, f"{what} {name}: expected 0, got max |g| {np.abs(g_gpu).max():.3e}"
        return
    rel = np.linalg.norm(g_gpu - g_ref) / np.linalg.norm(g_ref)
    assert rel <= GRAD_FRO, f"{what} {name}: relative Frobenius error {rel:.3e} > {GRAD_FRO}"


def to64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def run_gpu(q, k, v, do, scale, window=None):
    dev = torch.device("cuda")
    qd, kd, vd, dod = (x.to(dev) for x in (q, k, v, do))
    o, lse = attn.attn_fwd(qd, kd, vd, scale, window=window)
    dq, dk, dv = attn.attn_bwd(qd, kd, vd, o, lse, dod, scale, window=window)
    torch.cuda.synchronize()
    assert attn.get_device_error() == 0
    return o, lse, dq, dk, dv


def full_compare(w: Workload):
    q, k, v, do = make_inputs(w)
    win = w.window if w.window >= 0 else None
    o, lse, dq, dk, dv = run_gpu(q, k, v, do, w.scale, win)
    O_ref, LSE_ref = attn_ref.attention_forward(q, k, v, w.scale, window=win)
    dQ_ref, dK_ref, dV_ref, _ = attn_ref.attention_backward(q, k, v, do, w.scale, window=win)
    what = f"{w.name} B={w.B} H={w.H} Hkv={w.kv_heads} T={w.T} window={w.window}"
    check_o(to64(o), O_ref, what)
    check_lse(to64(lse), LSE_ref, what)
    check_grad(to64(dq), dQ_ref, "dQ", what)
    check_grad(to64(dk), dK_ref, "dK", what)
    check_grad(to64(dv), dV_ref, "dV", what)


def test_tiny_full():
    full_compare(WORKLOADS["tiny"])


# Ragged and edge sizes: T = 1 (O = V), tails inside the first tile, exactly one/two tiles, tails of 1 and
# 63 rows past a tile boundary, several heads and batches. Each spans the kernels' tiles and tails.
EDGE_SHAPES = [(1, 1, 1), (1, 1, 7), (2, 3, 64), (1, 2, 100), (1, 1, 128), (1, 2, 129), (2, 1, 191),
               (1, 1, 256), (1, 2, 383), (3, 2, 513)]


@pytest.mark.parametrize("B,H,T", EDGE_SHAPES, ids=[f"B{b}H{h}T{t}" for b, h, t in EDGE_SHAPES])
def test_edge_shapes_full(B, H, T):
    full_compare(Workload(f"edge", B=B, H=H, T=T, seed=T))


@pytest.mark.parametrize("prescale", [3.0, 6.0])
def test_peaky_rows_exercise_rescaling(prescale):
    """Q and K scaled up so softmax rows are peaky and the running max jumps by more than 2^8 within a row:
    the forward's lazy O rescaling runs, for some rows of a warp and not others."""
    full_compare(Workload(f"peaky{prescale}", B=1, H=2, T=640, seed=21, qk_prescale=prescale))


def test_T1_closed_form():
    w = Workload("T1", B=2, H=3, T=1, seed=5)
    q, k, v, do = make_inputs(w)
    o, lse, dq, dk, dv = run_gpu(q, k, v, do, w.scale)
    assert torch.equal(o.cpu(), v), "T = 1 must give O = V exactly"
    assert torch.equal(dv.cpu(), do), "T = 1 must give dV = dO exactly"
    # dQ = dK = 0 in closed form; the kernels leave only fp32 rounding of dP - Delta (a few 1e-4)
    assert float(dq.float().abs().max()) < 1e-2 and float(dk.float().abs().max()) < 1e-2


FULL = ["d12", "d20", "d24", "d26", "d26_T512", "d26_T1024", "d26_T4096"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled_slices(name):
    """The benchmark's shapes and launch; the oracle checks seeded (b, h) slices one by one."""
    w = WORKLOADS[name]
    q, k, v, do = make_inputs(w)
    o, lse, dq, dk, dv = run_gpu(q, k, v, do, w.scale)
    for (b, h) in sample_slices(w, k=5):  # (0, 0), (B-1, H-1) and three seeded mid-grid slices
        ref = attn_ref.slice_forward_backward(q, k, v, do, b, h, w.scale)
        what = f"{name} slice (b={b}, h={h})"
        check_o(to64(o[b, :, h]), ref["o"], what)
        check_lse(to64(lse[b, h]), ref["lse"], what)
        check_grad(to64(dq[b, :, h]), ref["dq"], "dQ", what)
        check_grad(to64(dk[b, :, h]), ref["dk"], "dK", what)
        check_grad(to64(dv[b, :, h]), ref["dv"], "dV", what)
    # Properties that hold at any size: finite everywhere, rows of dK and dV past no query are zero-free...
    for t in (o, dq, dk, dv):
        assert bool(torch.isfinite(t.float()).all())


# Grouped-query attention: k, v with H_kv heads, query head h reads head h // (H // H_kv).
GQA_SHAPES = [(1, 4, 2, 128), (2, 6, 2, 200), (1, 3, 1, 65), (1, 8, 4, 383), (2, 4, 1, 257), (1, 2, 2, 129)]


@pytest.mark.parametrize("B,H,Hkv,T", GQA_SHAPES, ids=[f"B{b}H{h}Hkv{hk}T{t}" for b, h, hk, t in GQA_SHAPES])
def test_gqa_full(B, H, Hkv, T):
    full_compare(Workload("gqa", B=B, H=H, T=T, Hkv=Hkv, seed=T + H))


def test_gqa_tiny_workload():
    full_compare(WORKLOADS["tiny_gqa"])


@pytest.mark.parametrize("name", ["d12_gqa", "d20_gqa"])
def test_gqa_full_size_sampled_groups(name):
    """Full-size grouped-query workloads: for sampled (b, key/value head) pairs, every query head of the group
    is checked as an oracle slice, and the shared head's dK, dV against the sum of the group's slices."""
    w = WORKLOADS[name]
    q, k, v, do = make_inputs(w)
    o, lse, dq, dk, dv = run_gpu(q, k, v, do, w.scale)
    G = w.H // w.kv_heads
    for (b, hk) in [(0, 0), (w.B - 1, w.kv_heads - 1)]:
        dk_ref, dv_ref = 0.0, 0.0
        for h in range(hk * G, (hk + 1) * G):
            ref = attn_ref.slice_forward_backward(q, k, v, do, b, h, w.scale)
            what = f"{name} slice (b={b}, h={h})"
            check_o(to64(o[b, :, h]), ref["o"], what)
            check_lse(to64(lse[b, h]), ref["lse"], what)
            check_grad(to64(dq[b, :, h]), ref["dq"], "dQ", what)
            dk_ref = dk_ref + ref["dk"]
            dv_ref = dv_ref + ref["dv"]
        check_grad(to64(dk[b, :, hk]), dk_ref, "dK", f"{name} kv head (b={b}, hk={hk})")
        check_grad(to64(dv[b, :, hk]), dv_ref, "dV", f"{name} kv head (b={b}, hk={hk})")
    for t in (o, dq, dk, dv):
        assert bool(torch.isfinite(t.float()).all())


# Sliding window: query i sees keys i - window .. i. Windows below, at and above a tile (64 or 128 rows), 0
# (each query sees only itself) and 1, ragged T, and combined with grouped-query attention.
WINDOW_SHAPES = [(1, 2, 2, 300, 100), (1, 1, 1, 257, 0), (1, 1, 1, 200, 1), (2, 2, 2, 513, 127), (1, 2, 2, 384, 128),
                 (1, 2, 1, 401, 129), (1, 4, 2, 640, 63), (1, 2, 2, 700, 200), (1, 1, 1, 130, 500)]


@pytest.mark.parametrize("B,H,Hkv,T,window", WINDOW_SHAPES,
                         ids=[f"B{b}H{h}Hkv{hk}T{t}W{w}" for b, h, hk, t, w in WINDOW_SHAPES])
def test_window_full(B, H, Hkv, T, window):
    full_compare(Workload("sw", B=B, H=H, T=T, Hkv=Hkv, window=window, seed=T + window))


def test_window_tiny_workload():
    full_compare(WORKLOADS["tiny_sw"])


def test_window_full_size_sampled_slices():
    """d20 shape with a 512-key window, at full size through the benchmark's launch; sampled slices."""
    w = WORKLOADS["d20_sw"]
    q, k, v, do = make_inputs(w)
    o, lse, dq, dk, dv = run_gpu(q, k, v, do, w.scale, w.window)
    for (b, h) in sample_slices(w, k=2):
        ref = attn_ref.slice_forward_backward(q, k, v, do, b, h, w.scale, window=w.window)
        what = f"d20_sw slice (b={b}, h={h})"
        check_o(to64(o[b, :, h]), ref["o"], what)
        check_lse(to64(lse[b, h]), ref["lse"], what)
        check_grad(to64(dq[b, :, h]), ref["dq"], "dQ", what)
        check_grad(to64(dk[b, :, h]), ref["dk"], "dK", what)
        check_grad(to64(dv[b, :, h]), ref["dv"], "dV", what)


def test_window_zero_gives_v_exactly():
    """window 0: every query sees only its own key, so O = V exactly and dV = dO exactly."""
    w = Workload("w0", B=1, H=2, T=300, window=0, seed=9)
    q, k, v, do = make_inputs(w)
    o, lse, dq, dk, dv = run_gpu(q, k, v, do, w.scale, 0)
    assert torch.equal(o.cpu(), v)
    assert torch.equal(dv.cpu(), do)


# Decode against a key/value cache (forward only).
DECODE_CASES = [("decode_tiny", None), ("small_mha", dict(B=2, H=2, Hkv=2, Tq=1, Tk=1000)),
                ("gqa_tq3", dict(B=3, H=8, Hkv=2, Tq=3, Tk=700)), ("short", dict(B=4, H=1, Hkv=1, Tq=4, Tk=5)),
                ("rows32", dict(B=1, H=16, Hkv=2, Tq=4, Tk=1300)), ("long", dict(B=1, H=2, Hkv=1, Tq=1, Tk=9000))]


@pytest.mark.parametrize("name,shape", DECODE_CASES, ids=[c[0] for c in DECODE_CASES])
def test_decode_full(name, shape):
    from workloads import DECODE_WORKLOADS, DecodeWorkload, make_decode_inputs
    w = DECODE_WORKLOADS[name] if shape is None else DecodeWorkload(name, seed=len(name), **shape)
    q, kc, vc, lens = make_decode_inputs(w)
    if name == "short":
        lens = torch.tensor([0, 1, 3, 5], dtype=torch.int32)  # empty cache, fewer keys than new queries, full
    dev = torch.device("cuda")
    o, lse = attn.attn_decode(q.to(dev), kc.to(dev), vc.to(dev), lens.to(dev), w.scale)
    torch.cuda.synchronize()
    O_ref, LSE_ref = attn_ref.decode_forward(q, kc, vc, lens.numpy(), w.scale)
    what = f"{name} lens={lens.tolist()[:6]}"
    check_o(to64(o), O_ref, what)
    finite = np.isfinite(LSE_ref)
    assert np.array_equal(np.isfinite(to64(lse)), finite), f"{what}: -inf LSE pattern differs"
    check_lse(to64(lse)[finite], LSE_ref[finite], what)
    assert np.all(to64(o)[np.broadcast_to(~finite.transpose(0, 2, 1)[..., None], O_ref.shape)] == 0)


DECODE_WINDOWS = [0, 1, 100, 127, 128, 129, 300, 5000]


@pytest.mark.parametrize("window", DECODE_WINDOWS)
def test_decode_window_full(window):
    """Sliding window in cached decode: ragged lengths, grouped heads, Tq = 3, windows below, at and above a
    128-key block and beyond the cache; every output against the oracle's end-aligned band."""
    from workloads import DecodeWorkload, make_decode_inputs
    w = DecodeWorkload("decode_sw", B=3, H=8, Hkv=2, Tq=3, Tk=1300, seed=41 + window)
    q, kc, vc, lens = make_decode_inputs(w)
    dev = torch.device("cuda")
    o, lse = attn.attn_decode(q.to(dev), kc.to(dev), vc.to(dev), lens.to(dev), w.scale, window=window)
    torch.cuda.synchronize()
    O_ref, LSE_ref = attn_ref.decode_forward(q, kc, vc, lens.numpy(), w.scale, window=window)
    what = f"decode window={window} lens={lens.tolist()}"
    check_o(to64(o), O_ref, what)
    finite = np.isfinite(LSE_ref)
    assert np.array_equal(np.isfinite(to64(lse)), finite), f"{what}: -inf LSE pattern differs"
    check_lse(to64(lse)[finite], LSE_ref[finite], what)


def test_decode_window_long_cache_single_token():
    """One new token per sequence against 9000 cached keys with a 1000-key window: the chunks cover only the
    band, and window >= the cache length equals no window bit for bit."""
    from workloads import DecodeWorkload, make_decode_inputs
    w = DecodeWorkload("decode_sw_long", B=2, H=4, Hkv=1, Tq=1, Tk=9000, seed=77)
    q, kc, vc, lens = make_decode_inputs(w)
    dev = torch.device("cuda")
    args = (q.to(dev), kc.to(dev), vc.to(dev), lens.to(dev), w.scale)
    o, lse = attn.attn_decode(*args, window=1000)
    torch.cuda.synchronize()
    O_ref, LSE_ref = attn_ref.decode_forward(q, kc, vc, lens.numpy(), w.scale, window=1000)
    check_o(to64(o), O_ref, "decode window=1000 Tk=9000")
    check_lse(to64(lse), LSE_ref, "decode window=1000 Tk=9000")
    o_all, lse_all = attn.attn_decode(*args)
    o_big, lse_big = attn.attn_decode(*args, window=9000)
    assert torch.equal(o_all, o_big) and torch.equal(lse_all, lse_big)


@pytest.mark.parametrize("window", [None, 1000])
def test_decode_many_sequences_every_chunk_once(window):
    """600 one-head sequences against a 4352-key cache (34 blocks of 128): one chunk per sequence, so the CTAs'
    longest-first order sorts 600 (sequence, chunk) pairs over 35 block counts, several 32-wide windows of
    each. Six seeded sequences hold random keys and values and go to the oracle; every other cache is zero, so
    its output is exactly 0 and its LSE ln(keys seen) (-inf for an empty cache). o and lse start as NaN: every
    (sequence, chunk) must be computed, and computed once."""
    B, Tk, D = 600, 4352, 128
    g = torch.Generator(device="cpu")
    g.manual_seed(4352)
    lens = torch.randint(1, Tk + 1, (B,), generator=g, dtype=torch.int64).to(torch.int32)
    lens[3], lens[4], lens[5] = 0, Tk, 1
    q = torch.randn((B, 1, 1, D), generator=g).to(torch.bfloat16)
    picks = [0, 3, 4, 5, 311, B - 1]
    dev = torch.device("cuda")
    kc = torch.zeros((B, Tk, 1, D), dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    cpu_k, cpu_v = {}, {}
    for b in picks:
        cpu_k[b] = torch.zeros((1, Tk, 1, D), dtype=torch.bfloat16)
        cpu_v[b] = torch.zeros((1, Tk, 1, D), dtype=torch.bfloat16)
        L = int(lens[b])
        cpu_k[b][0, :L] = torch.randn((L, 1, D), generator=g).to(torch.bfloat16)
        cpu_v[b][0, :L] = torch.randn((L, 1, D), generator=g).to(torch.bfloat16)
        kc[b].copy_(cpu_k[b][0])
        vc[b].copy_(cpu_v[b][0])
    o = torch.full((B, 1, 1, D), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((B, 1, 1), float("nan"), dtype=torch.float32, device=dev)
    scale = D ** -0.5
    attn.attn_decode(q.to(dev), kc, vc, lens.to(dev), scale, o=o, lse=lse, window=window)
    torch.cuda.synchronize()
    assert attn.load_library().attn_decode_kernels(B, 1, 1, 1, Tk, D, -1 if window is None else window) == 1
    o64, lse64 = to64(o), to64(lse)
    for b in picks:
        O_ref, LSE_ref = attn_ref.decode_forward(q[b:b + 1], cpu_k[b], cpu_v[b], lens[b:b + 1].numpy(), scale,
                                                 window=window)
        what = f"decode B=600 b={b} L={int(lens[b])}"
        check_o(o64[b:b + 1], O_ref, what)
        finite = np.isfinite(LSE_ref)
        assert np.array_equal(np.isfinite(lse64[b:b + 1]), finite), f"{what}: -inf LSE pattern differs"
        check_lse(lse64[b:b + 1][finite], LSE_ref[finite], what)
    rest = np.array([b for b in range(B) if b not in picks])
    seen = lens.numpy()[rest].astype(np.float64)
    if window is not None:
        seen = np.minimum(seen, window + 1)
    assert np.all(o64[rest] == 0), "a zero cache must give o = 0 exactly (NaN: a chunk was never computed)"
    check_lse(lse64[rest, 0, 0], np.log(seen), "decode B=600 zero caches")


def test_decode_one_cta_per_unit_beyond_the_walk_limit():
    """1000 sequences of 10 heads against a 128-key cache: 10,000 (sequence, head) units, more than a persistent
    CTA per SM lists (64 each), so the grid takes one CTA per unit. Three seeded sequences go to the oracle;
    every other cache is zero (o = 0 exactly, LSE = ln(keys seen)); o and lse start as NaN."""
    B, H, Tk, D = 1000, 10, 128, 128
    g = torch.Generator(device="cpu")
    g.manual_seed(10000)
    lens = torch.randint(1, Tk + 1, (B,), generator=g, dtype=torch.int64).to(torch.int32)
    q = torch.randn((B, 1, H, D), generator=g).to(torch.bfloat16)
    picks = [0, 517, B - 1]
    dev = torch.device("cuda")
    kc = torch.zeros((B, Tk, H, D), dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    cpu_k, cpu_v = {}, {}
    for b in picks:
        cpu_k[b] = torch.randn((1, Tk, H, D), generator=g).to(torch.bfloat16)
        cpu_v[b] = torch.randn((1, Tk, H, D), generator=g).to(torch.bfloat16)
        kc[b].copy_(cpu_k[b][0])
        vc[b].copy_(cpu_v[b][0])
    o = torch.full((B, 1, H, D), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((B, H, 1), float("nan"), dtype=torch.float32, device=dev)
    scale = D ** -0.5
    attn.attn_decode(q.to(dev), kc, vc, lens.to(dev), scale, o=o, lse=lse)
    torch.cuda.synchronize()
    o64, lse64 = to64(o), to64(lse)
    for b in picks:
        O_ref, LSE_ref = attn_ref.decode_forward(q[b:b + 1], cpu_k[b], cpu_v[b], lens[b:b + 1].numpy(), scale)
        check_o(o64[b:b + 1], O_ref, f"decode B=1000 b={b}")
        check_lse(lse64[b:b + 1], LSE_ref, f"decode B=1000 b={b}")
    rest = np.array([b for b in range(B) if b not in picks])
    assert np.all(o64[rest] == 0), "a zero cache must give o = 0 exactly (NaN: a unit was never computed)"
    seen = np.broadcast_to(lens.numpy()[rest].astype(np.float64)[:, None, None], lse64[rest].shape)
    check_lse(lse64[rest], np.log(seen), "decode B=1000 zero caches")


@pytest.mark.parametrize("name", ["decode_d20", "decode_d20_gqa", "decode_d20_sw"])
def test_decode_full_size_sampled(name):
    """The benchmark's decode workloads (64 sequences, d20 heads, ragged lengths up to 2048), oracle on samples.
    decode_d20 and decode_d20_sw take one cache chunk per (sequence, head), whose kernel writes o and lse itself;
    decode_d20_gqa splits the cache and merges the chunks in a second kernel."""
    from workloads import DECODE_WORKLOADS, make_decode_inputs
    w = DECODE_WORKLOADS[name]
    win = w.window if w.window >= 0 else None
    q, kc, vc, lens = make_decode_inputs(w)
    dev = torch.device("cuda")
    o, lse = attn.attn_decode(q.to(dev), kc.to(dev), vc.to(dev), lens.to(dev), w.scale, window=win)
    torch.cuda.synchronize()
    for b in (0, 17, w.B - 1):
        O_ref, LSE_ref = attn_ref.decode_forward(q[b:b + 1], kc[b:b + 1], vc[b:b + 1], lens[b:b + 1].numpy(), w.scale,
                                                 window=win)
        check_o(to64(o[b:b + 1]), O_ref, f"{name} b={b}")
        check_lse(to64(lse[b:b + 1]), LSE_ref, f"{name} b={b}")


def test_causality_on_gpu():
    """Perturbing q/k/v after position t leaves O and LSE at positions <= t bit-identical."""
    w = Workload("causal", B=2, H=2, T=300, seed=9)
    q, k, v, _ = make_inputs(w, need_grad_input=False)
    dev = torch.device("cuda")
    o1, l1 = attn.attn_fwd(q.to(dev), k.to(dev), v.to(dev), w.scale)
    t = 150
    q2, k2, v2 = q.clone(), k.clone(), v.clone()
    for x in (q2, k2, v2):
        x[:, t + 1:] = torch.randn_like(x[:, t + 1:].float()).to(torch.bfloat16) * 3
    o2, l2 = attn.attn_fwd(q2.to(dev), k2.to(dev), v2.to(dev), w.scale)
    assert torch.equal(o1[:, :t + 1], o2[:, :t + 1])
    assert torch.equal(l1[:, :, :t + 1], l2[:, :, :t + 1])


def test_key_shift_invariance_d24_recipe():
    """Adding one vector to every key leaves O unchanged and shifts LSE by scale * q . b (d24's input recipe)."""
    w = Workload("shift", B=1, H=2, T=512, seed=3)
    q, k, v, _ = make_inputs(w, need_grad_input=False)
    bias = torch.randn(w.D, generator=torch.Generator().manual_seed(7))
    k2 = (k.float() + bias).to(torch.bfloat16)
    dev = torch.device("cuda")
    o1, l1 = attn.attn_fwd(q.to(dev), k.to(dev), v.to(dev), w.scale)
    o2, l2 = attn.attn_fwd(q.to(dev), k2.to(dev), v.to(dev), w.scale)
    ref_o, ref_l = attn_ref.attention_forward(q, k2, v, w.scale)
    check_o(to64(o2), ref_o, "shifted keys")
    check_lse(to64(l2), ref_l, "shifted keys")
    check_o(to64(o2), to64(o1), "shift invariance")


def test_repeated_calls_are_deterministic_forward():
    w = Workload("det", B=2, H=3, T=777, seed=4)
    q, k, v, _ = make_inputs(w, need_grad_input=False)
    dev = torch.device("cuda")
    a = attn.attn_fwd(q.to(dev), k.to(dev), v.to(dev), w.scale)
    b = attn.attn_fwd(q.to(dev), k.to(dev), v.to(dev), w.scale)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_autograd_wrapper_matches_oracle():
    w = Workload("autograd", B=1, H=2, T=200, seed=12)
    q, k, v, do = make_inputs(w)
    dev = torch.device("cuda")
    qd, kd, vd = (x.to(dev).requires_grad_() for x in (q, k, v))
    out = attn.causal_attention(qd, kd, vd)
    out.backward(do.to(dev))
    dQ_ref, dK_ref, dV_ref, _ = attn_ref.attention_backward(q, k, v, do, w.scale)
    check_grad(to64(qd.grad), dQ_ref, "dQ")
    check_grad(to64(kd.grad), dK_ref, "dK")
    check_grad(to64(vd.grad), dV_ref, "dV")


def test_argument_errors_on_gpu():
    dev = torch.device("cuda")
    q = torch.zeros(1, 64, 1, 128, dtype=torch.bfloat16, device=dev)
    lib = attn.load_library()
    lse = torch.empty(1, 1, 64, device=dev)
    o = torch.empty_like(q)
    # misaligned output pointer
    assert lib.attn_fwd(q.data_ptr(), q.data_ptr(), q.data_ptr(), o.data_ptr() + 2, lse.data_ptr(), 1, 1, 64, 128,
                        0.1, None) == 3
    ws = torch.empty(attn.attn_bwd_workspace_bytes(1, 1, 64, 128) - 256, dtype=torch.uint8, device=dev)
    with pytest.raises(attn.AttnError):
        attn.attn_bwd(q, q, q, q, lse, q, 0.1, workspace=ws)


def test_bounded_wait_reports_timeout():
    """A kernel that waits on a barrier nothing completes gives up after its limit and reports the site."""
    attn.clear_device_error()
    attn.selftest_wait_timeout(2_000_000)  # 2 ms
    torch.cuda.synchronize()
    word = attn.get_device_error()
    assert word == (0x7F << 8) | 1
    attn.clear_device_error()
    assert attn.get_device_error() == 0
    # the context is still usable afterwards
    test_tiny_full()
