"""Pins for the float64 oracle, each tied to something other than the oracle itself.

The pages define the operation only as ``flash_attn_func(q, k, v, causal=True)`` (apidog "Train your own
ChatGPT", section 5), with a PyTorch SDPA fallback on other hardware (same section). So the oracle is pinned
by: a hand-derived worked example (tests/golden), closed forms (T = 1, Q = 0, equal keys), invariants
(softmax rows, causality, key shift), torch's own float64 SDPA and autograd (the fallback the pages name), and
central finite differences. The last test plants mistakes in a copy of the oracle and checks that these pins
catch each one.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import attn_ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example_T3.txt")


def load_golden(path=GOLDEN):
    cases, cur = {}, None
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            if key == "case":
                cur = cases.setdefault(vals[0], {})
            else:
                cur[key] = np.array([float(x) for x in vals])
    return cases


def rand_qkvdo(T, D, seed, B=1, H=1):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal((B, T, H, D)) for _ in range(4)]


# ---------------------------------------------------------------------------------------------------------
# Pin checks, parameterised by the implementation so that the mutation test can reuse them.
# An implementation is a pair (fwd(q,k,v,s) -> (O, lse, P), bwd(q,k,v,do,s) -> (dq, dk, dv, delta)) per head.

ORACLE = (attn_ref.head_forward, lambda q, k, v, do, s: attn_ref.head_backward(q, k, v, do, s))


def check_golden(impl):
    fwd, bwd = impl
    for name, c in load_golden().items():
        T = len(c["lse"])
        D = len(c["q"]) // T
        q, k, v, do = (c[n].reshape(T, D) for n in ("q", "k", "v", "do"))
        s = float(c["scale"][0])
        O, lse, _ = fwd(q, k, v, s)
        dq, dk, dv, delta = bwd(q, k, v, do, s)
        np.testing.assert_allclose(O, c["o"].reshape(T, D), rtol=0, atol=1e-14, err_msg=f"{name}: O")
        np.testing.assert_allclose(lse, c["lse"], rtol=0, atol=1e-14, err_msg=f"{name}: lse")
        np.testing.assert_allclose(delta, c["delta"], rtol=0, atol=1e-14, err_msg=f"{name}: delta")
        np.testing.assert_allclose(dv, c["dv"].reshape(T, D), rtol=0, atol=1e-14, err_msg=f"{name}: dv")
        np.testing.assert_allclose(dq, c["dq"].reshape(T, D), rtol=0, atol=1e-14, err_msg=f"{name}: dq")
        np.testing.assert_allclose(dk, c["dk"].reshape(T, D), rtol=0, atol=1e-14, err_msg=f"{name}: dk")


def check_softmax_rows(impl, T=37, D=16, seed=0):
    fwd, _ = impl
    q, k, v, _ = (x[0, :, 0] for x in rand_qkvdo(T, D, seed))
    _, _, P = fwd(q, k, v, 1 / math.sqrt(D))
    assert np.all(P >= 0)
    assert np.all(P[np.triu_indices(T, 1)] == 0), "weight on a future key"
    np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-12)


def check_causality(impl, T=29, D=8, seed=1):
    fwd, _ = impl
    q, k, v, _ = (x[0, :, 0] for x in rand_qkvdo(T, D, seed))
    s = 1 / math.sqrt(D)
    O, lse, _ = fwd(q, k, v, s)
    rng = np.random.default_rng(seed + 100)
    for t in (0, 5, T - 2):
        q2, k2, v2 = q.copy(), k.copy(), v.copy()
        for a in (q2, k2, v2):
            a[t + 1:] += 10 * rng.standard_normal(a[t + 1:].shape)
        O2, lse2, _ = fwd(q2, k2, v2, s)
        np.testing.assert_array_equal(O2[:t + 1], O[:t + 1])
        np.testing.assert_array_equal(lse2[:t + 1], lse[:t + 1])


def check_T1(impl, D=8, seed=2):
    fwd, bwd = impl
    q, k, v, do = (x[0, :, 0] for x in rand_qkvdo(1, D, seed))
    s = 0.37
    O, lse, _ = fwd(q, k, v, s)
    np.testing.assert_allclose(O, v, rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, [s * float(q[0] @ k[0])], rtol=1e-15, atol=1e-15)
    dq, dk, dv, _ = bwd(q, k, v, do, s)
    np.testing.assert_allclose(dv, do, rtol=0, atol=1e-15)
    np.testing.assert_allclose(dq, 0, atol=1e-15)
    np.testing.assert_allclose(dk, 0, atol=1e-15)


def check_zero_query(impl, T=23, D=8, seed=3):
    fwd, _ = impl
    _, k, v, _ = (x[0, :, 0] for x in rand_qkvdo(T, D, seed))
    q = np.zeros((T, D))
    O, lse, _ = fwd(q, k, v, 0.5)
    prefix_mean = np.cumsum(v, axis=0) / np.arange(1, T + 1)[:, None]
    np.testing.assert_allclose(O, prefix_mean, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse, np.log(np.arange(1, T + 1)), rtol=1e-14, atol=1e-14)


def check_equal_keys(impl, T=19, D=8, seed=4):
    fwd, _ = impl
    q, k, v, _ = (x[0, :, 0] for x in rand_qkvdo(T, D, seed))
    k = np.repeat(k[:1], T, axis=0)
    O, _, _ = fwd(q, k, v, 0.3)
    prefix_mean = np.cumsum(v, axis=0) / np.arange(1, T + 1)[:, None]
    np.testing.assert_allclose(O, prefix_mean, rtol=1e-13, atol=1e-14)


def check_key_shift(impl, T=31, D=8, seed=5):
    """Adding one vector b to every key shifts logit row i by s q_i . b: P, O unchanged, LSE shifted."""
    fwd, bwd = impl
    q, k, v, do = (x[0, :, 0] for x in rand_qkvdo(T, D, seed))
    b = np.random.default_rng(seed).standard_normal(D)
    s = 1 / math.sqrt(D)
    O, lse, _ = fwd(q, k, v, s)
    O2, lse2, _ = fwd(q, k + b, v, s)
    np.testing.assert_allclose(O2, O, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse2, lse + s * (q @ b), rtol=1e-12, atol=1e-12)
    dq, dk, dv, _ = bwd(q, k, v, do, s)
    dq2, dk2, dv2, _ = bwd(q, k + b, v, do, s)
    np.testing.assert_allclose(dv2, dv, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(dk2, dk, rtol=1e-11, atol=1e-11)
    # dQ picks up s * sum_j dS_ij b = 0, since each row of dS sums to zero.
    np.testing.assert_allclose(dq2, dq, rtol=1e-11, atol=1e-11)


def check_torch_sdpa(impl, T=45, D=16, seed=6):
    """Agreement with torch's float64 CPU scaled_dot_product_attention and its autograd."""
    fwd, bwd = impl
    q, k, v, do = (x[0, :, 0] for x in rand_qkvdo(T, D, seed))
    s = 1 / math.sqrt(D)
    tq, tk, tv = (torch.tensor(x[None, None], dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=s)
    (to * torch.tensor(do[None, None])).sum().backward()
    O, _, _ = fwd(q, k, v, s)
    dq, dk, dv, _ = bwd(q, k, v, do, s)
    np.testing.assert_allclose(O, to[0, 0].detach().numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dq, tq.grad[0, 0].numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad[0, 0].numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad[0, 0].numpy(), rtol=1e-11, atol=1e-12)


def check_finite_differences(impl, T=6, D=5, seed=7, h=1e-6):
    """Central differences of f = sum(dO * O) against the analytic gradient."""
    fwd, bwd = impl
    q, k, v, do = (x[0, :, 0] for x in rand_qkvdo(T, D, seed))
    s = 0.45

    def f(q_, k_, v_):
        return float((do * fwd(q_, k_, v_, s)[0]).sum())

    dq, dk, dv, _ = bwd(q, k, v, do, s)
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        num = np.zeros_like(grad)
        for idx in np.ndindex(grad.shape):
            args_p = [q.copy(), k.copy(), v.copy()]
            args_m = [q.copy(), k.copy(), v.copy()]
            args_p[which][idx] += h
            args_m[which][idx] -= h
            num[idx] = (f(*args_p) - f(*args_m)) / (2 * h)
        rel = np.linalg.norm(num - grad) / max(np.linalg.norm(grad), 1e-30)
        assert rel < 1e-6, f"finite differences, input {which}: relative error {rel:.3e}"


def check_delta_identity(impl, T=33, D=8, seed=8):
    fwd, bwd = impl
    q, k, v, do = (x[0, :, 0] for x in rand_qkvdo(T, D, seed))
    s = 1 / math.sqrt(D)
    _, _, P = fwd(q, k, v, s)
    _, _, _, delta = bwd(q, k, v, do, s)
    dP = do @ v.T
    np.testing.assert_allclose(delta, (P * dP).sum(axis=1), rtol=1e-12, atol=1e-12)


ALL_PINS = [check_golden, check_softmax_rows, check_causality, check_T1, check_zero_query, check_equal_keys,
            check_key_shift, check_torch_sdpa, check_finite_differences, check_delta_identity]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(ORACLE)


# ---------------------------------------------------------------------------------------------------------
# The full-tensor entry points agree with the per-head ones and with torch on a batched [B, T, H, D] case.

def test_full_tensor_entry_points_match_torch():
    B, T, H, D = 2, 40, 3, 16
    q, k, v, do = rand_qkvdo(T, D, 11, B=B, H=H)
    s = 1 / math.sqrt(D)
    O, LSE = attn_ref.attention_forward(q, k, v, s)
    dQ, dK, dV, delta = attn_ref.attention_backward(q, k, v, do, s)
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64).transpose(1, 2).requires_grad_() for x in (q, k, v))
    to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=s)
    (to * torch.tensor(do).transpose(1, 2)).sum().backward()
    np.testing.assert_allclose(O, to.transpose(1, 2).detach().numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dQ, tq.grad.transpose(1, 2).numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dK, tk.grad.transpose(1, 2).numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dV, tv.grad.transpose(1, 2).numpy(), rtol=1e-11, atol=1e-12)
    # LSE against torch.logsumexp of the masked, scaled logits.
    S = s * torch.einsum("bhid,bhjd->bhij", tq.detach(), tk.detach())
    S = S.masked_fill(~torch.ones(T, T, dtype=torch.bool).tril(), float("-inf"))
    np.testing.assert_allclose(LSE, torch.logsumexp(S, dim=-1).numpy(), rtol=1e-13, atol=1e-13)
    # Slices are independent: the slice entry point returns the same numbers.
    sl = attn_ref.slice_forward_backward(q, k, v, do, 1, 2, s)
    np.testing.assert_allclose(sl["o"], O[1, :, 2], rtol=0, atol=1e-15)
    np.testing.assert_allclose(sl["dk"], dK[1, :, 2], rtol=0, atol=1e-15)
    np.testing.assert_allclose(sl["delta"], delta[1, 2], rtol=0, atol=1e-15)


# ---------------------------------------------------------------------------------------------------------
# Grouped-query attention: k, v with H_kv heads, query head h reads head h // (H // H_kv).

def _torch_gqa(q, k, v, do, s):
    """torch's float64 SDPA with its own grouped-query mode (enable_gqa) and autograd."""
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64).transpose(1, 2).requires_grad_() for x in (q, k, v))
    to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=s, enable_gqa=True)
    (to * torch.tensor(do).transpose(1, 2)).sum().backward()
    return [x.transpose(1, 2).detach().numpy() for x in (to, tq.grad, tk.grad, tv.grad)]


@pytest.mark.parametrize("H,Hkv", [(4, 2), (6, 2), (3, 1), (4, 4)])
def test_gqa_matches_torch_enable_gqa(H, Hkv):
    B, T, D = 2, 33, 16
    rng = np.random.default_rng(7 + H + Hkv)
    q, do = rng.standard_normal((B, T, H, D)), rng.standard_normal((B, T, H, D))
    k, v = rng.standard_normal((B, T, Hkv, D)), rng.standard_normal((B, T, Hkv, D))
    s = 1 / math.sqrt(D)
    O, LSE = attn_ref.attention_forward(q, k, v, s)
    dQ, dK, dV, _ = attn_ref.attention_backward(q, k, v, do, s)
    to, gq, gk, gv = _torch_gqa(q, k, v, do, s)
    np.testing.assert_allclose(O, to, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dQ, gq, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dK, gk, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dV, gv, rtol=1e-11, atol=1e-12)
    # The slice entry point reads the group's key/value head; its dk is that head's contribution.
    h = H - 1
    sl = attn_ref.slice_forward_backward(q, k, v, do, 1, h, s)
    np.testing.assert_allclose(sl["o"], O[1, :, h], rtol=0, atol=1e-15)
    np.testing.assert_allclose(sl["dq"], dQ[1, :, h], rtol=0, atol=1e-15)


def test_gqa_key_gradient_by_finite_differences():
    """dK of a shared key/value head is the sum over its query heads: checked by central differences of
    L = sum(O * dO) with respect to single key and value entries."""
    B, T, H, Hkv, D = 1, 6, 4, 2, 4
    rng = np.random.default_rng(3)
    q, do = rng.standard_normal((B, T, H, D)), rng.standard_normal((B, T, H, D))
    k, v = rng.standard_normal((B, T, Hkv, D)), rng.standard_normal((B, T, Hkv, D))
    s = 0.7
    _, dK, dV, _ = attn_ref.attention_backward(q, k, v, do, s)
    loss = lambda kk, vv: float((attn_ref.attention_forward(q, kk, vv, s)[0] * do).sum())
    eps = 1e-6
    for (t, hk, d) in [(0, 0, 1), (2, 1, 3), (5, 1, 0), (3, 0, 2)]:
        kp, km = k.copy(), k.copy()
        kp[0, t, hk, d] += eps
        km[0, t, hk, d] -= eps
        assert abs((loss(kp, v) - loss(km, v)) / (2 * eps) - dK[0, t, hk, d]) < 1e-7
        vp, vm = v.copy(), v.copy()
        vp[0, t, hk, d] += eps
        vm[0, t, hk, d] -= eps
        assert abs((loss(k, vp) - loss(k, vm)) / (2 * eps) - dV[0, t, hk, d]) < 1e-7


def test_gqa_pin_catches_a_wrong_head_mapping():
    """Interleaved sharing (h % H_kv) instead of consecutive sharing is caught by the torch pin."""
    B, T, H, Hkv, D = 1, 20, 4, 2, 8
    rng = np.random.default_rng(5)
    q, do = rng.standard_normal((B, T, H, D)), rng.standard_normal((B, T, H, D))
    k, v = rng.standard_normal((B, T, Hkv, D)), rng.standard_normal((B, T, Hkv, D))
    s = 1 / math.sqrt(D)
    wrong = np.stack([attn_ref.head_forward(q[0, :, h], k[0, :, h % Hkv], v[0, :, h % Hkv], s)[0] for h in range(H)],
                     axis=1)[None]
    to = _torch_gqa(q, k, v, do, s)[0]
    assert np.abs(wrong - to).max() > 1e-3
    with pytest.raises(ValueError):
        attn_ref.attention_forward(q, k[:, :, :1].repeat(3, axis=2), v[:, :, :1].repeat(3, axis=2), s)


# ---------------------------------------------------------------------------------------------------------
# Sliding window: query i sees keys i - window .. i.

def _band(T, window):
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    return (j <= i) & (j >= i - window)


@pytest.mark.parametrize("T,window,H,Hkv", [(37, 5, 2, 2), (40, 0, 2, 2), (33, 16, 4, 2), (50, 1, 3, 1)])
def test_window_matches_torch_with_band_mask(T, window, H, Hkv):
    """torch's float64 SDPA given the band as an explicit boolean mask (and enable_gqa), with autograd."""
    B, D = 2, 16
    rng = np.random.default_rng(T + window)
    q, do = rng.standard_normal((B, T, H, D)), rng.standard_normal((B, T, H, D))
    k, v = rng.standard_normal((B, T, Hkv, D)), rng.standard_normal((B, T, Hkv, D))
    s = 1 / math.sqrt(D)
    O, LSE = attn_ref.attention_forward(q, k, v, s, window=window)
    dQ, dK, dV, _ = attn_ref.attention_backward(q, k, v, do, s, window=window)
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64).transpose(1, 2).requires_grad_() for x in (q, k, v))
    to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=_band(T, window), scale=s,
                                                          enable_gqa=True)
    (to * torch.tensor(do).transpose(1, 2)).sum().backward()
    np.testing.assert_allclose(O, to.transpose(1, 2).detach().numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dQ, tq.grad.transpose(1, 2).numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dK, tk.grad.transpose(1, 2).numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dV, tv.grad.transpose(1, 2).numpy(), rtol=1e-11, atol=1e-12)
    # LSE against torch.logsumexp over the band.
    kk = np.repeat(k, H // Hkv, axis=2)
    S = s * np.einsum("bihd,bjhd->bhij", q, kk)
    S = np.where(_band(T, window).numpy(), S, -np.inf)
    np.testing.assert_allclose(LSE, torch.logsumexp(torch.tensor(S), dim=-1).numpy(), rtol=1e-13, atol=1e-13)


def test_window_closed_forms():
    """window >= T-1 is plain causal attention; window 0 leaves each query only itself: O = V exactly and
    LSE = scale * q.k of the row's own key."""
    T, D = 30, 8
    q, k, v, do = rand_qkvdo(T, D, 4)
    s = 0.4
    O, LSE = attn_ref.attention_forward(q, k, v, s)
    Ow, LSEw = attn_ref.attention_forward(q, k, v, s, window=T - 1)
    np.testing.assert_array_equal(O, Ow)
    np.testing.assert_array_equal(LSE, LSEw)
    O0, LSE0 = attn_ref.attention_forward(q, k, v, s, window=0)
    np.testing.assert_allclose(O0, v, rtol=0, atol=1e-15)
    np.testing.assert_allclose(LSE0[0, 0], s * (q[0, :, 0] * k[0, :, 0]).sum(axis=1), rtol=1e-14, atol=1e-14)
    with pytest.raises(ValueError):
        attn_ref.attention_forward(q, k, v, s, window=-2)


@pytest.mark.parametrize("kind", ["left_edge_excluded", "one_key_wider", "window_ignored"])
def test_window_pin_catches_a_wrong_band(monkeypatch, kind):
    """Planted mistakes in the band the oracle builds: the torch band-mask pin must fail on each."""
    def mutated(T, window=None):
        i, j = np.arange(T)[:, None], np.arange(T)[None, :]
        if window is None or kind == "window_ignored":
            return j <= i
        lo = {"left_edge_excluded": i - window + 1, "one_key_wider": i - window - 1}[kind]
        return (j <= i) & (j >= lo)
    monkeypatch.setattr(attn_ref, "causal_mask", mutated)
    with pytest.raises(AssertionError):
        test_window_matches_torch_with_band_mask(37, 5, 2, 2)


def test_window_gradients_by_finite_differences():
    T, D, window = 9, 4, 3
    q, k, v, do = rand_qkvdo(T, D, 8)
    s = 0.6
    dQ, dK, dV, _ = attn_ref.attention_backward(q, k, v, do, s, window=window)
    loss = lambda qq, kk, vv: float((attn_ref.attention_forward(qq, kk, vv, s, window=window)[0] * do).sum())
    eps = 1e-6
    for name, x, g in (("q", q, dQ), ("k", k, dK), ("v", v, dV)):
        for (t, d) in [(0, 0), (4, 2), (8, 3), (6, 1)]:
            xp, xm = x.copy(), x.copy()
            xp[0, t, 0, d] += eps
            xm[0, t, 0, d] -= eps
            args_p = [xp if n == name else y for n, y in (("q", q), ("k", k), ("v", v))]
            args_m = [xm if n == name else y for n, y in (("q", q), ("k", k), ("v", v))]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - g[0, t, 0, d]) < 1e-7, (name, t, d)


# ---------------------------------------------------------------------------------------------------------
# Decode against a key/value cache: query i of Tq sits at position L - Tq + i.

def decode_pin_whole_sequence(f):
    """Tq = L: the new queries are the whole sequence, so decode is the causal training forward."""
    B, T, H, Hkv, D = 2, 21, 4, 2, 8
    rng = np.random.default_rng(11)
    q = rng.standard_normal((B, T, H, D))
    k, v = rng.standard_normal((B, T, Hkv, D)), rng.standard_normal((B, T, Hkv, D))
    s = 0.3
    O, LSE = f(q, k, v, [T, T], s)
    O2, LSE2 = attn_ref.attention_forward(q, k, v, s)
    np.testing.assert_allclose(O, O2, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(LSE, LSE2, rtol=1e-13, atol=1e-13)


def decode_pin_torch(f):
    """Ragged cache lengths, spare cache rows filled with garbage (never read), Tq = 3: each sequence equals
    torch's float64 SDPA on its valid cache with the end-aligned causal mask (and enable_gqa)."""
    B, Tq, H, Hkv, Tk, D = 3, 3, 6, 2, 40, 16
    rng = np.random.default_rng(12)
    q = rng.standard_normal((B, Tq, H, D))
    kc, vc = rng.standard_normal((B, Tk, Hkv, D)), rng.standard_normal((B, Tk, Hkv, D))
    lens = [40, 17, 3]
    s = 1 / math.sqrt(D)
    O, LSE = f(q, kc, vc, lens, s)
    for b, L in enumerate(lens):
        tq = torch.tensor(q[b:b + 1]).transpose(1, 2)
        tk, tv = (torch.tensor(x[b:b + 1, :L]).transpose(1, 2) for x in (kc, vc))
        pos = torch.arange(L - Tq, L)[:, None]
        mask = torch.arange(L)[None, :] <= pos
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=s, enable_gqa=True)
        np.testing.assert_allclose(O[b:b + 1], ref.transpose(1, 2).numpy(), rtol=1e-12, atol=1e-12)
    # garbage past the lengths does not matter
    kc2, vc2 = kc.copy(), vc.copy()
    kc2[1, 17:] = 1e6
    vc2[2, 3:] = np.nan
    O2, _ = f(q, kc2, vc2, lens, s)
    np.testing.assert_array_equal(O, O2)


def decode_pin_closed_forms(f):
    """Tq = 1 sees the whole valid cache (softmax over all L keys, LSE its log-sum-exp); a query before the
    first key (L < Tq) returns 0 with LSE -inf; L = 1 returns the one value."""
    B, Tk, H, D = 2, 9, 1, 4
    rng = np.random.default_rng(13)
    q = rng.standard_normal((B, 2, H, D))
    kc, vc = rng.standard_normal((B, Tk, H, D)), rng.standard_normal((B, Tk, H, D))
    s = 0.5
    O, LSE = f(q[:, :1], kc, vc, [9, 1], s)
    sc = s * kc[0, :, 0] @ q[0, 0, 0]
    p = np.exp(sc - sc.max()) / np.exp(sc - sc.max()).sum()
    np.testing.assert_allclose(O[0, 0, 0], p @ vc[0, :, 0], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(LSE[0, 0, 0], np.log(np.exp(sc).sum()), rtol=1e-13)
    np.testing.assert_allclose(O[1, 0, 0], vc[1, 0, 0], rtol=0, atol=1e-15)
    O2, LSE2 = f(q, kc, vc, [9, 1], s)   # Tq = 2, second sequence has one key
    assert np.all(O2[1, 0, 0] == 0) and LSE2[1, 0, 0] == -np.inf
    np.testing.assert_allclose(O2[1, 1, 0], vc[1, 0, 0], rtol=0, atol=1e-15)


def decode_pin_window_torch(f):
    """Sliding window in decode: ragged lengths, Tq = 3, grouped heads, windows below, at and above the
    lengths: each sequence equals torch's float64 SDPA with the band p - W <= j <= p aligned to the end of
    the cache, given as an explicit mask."""
    B, Tq, H, Hkv, Tk, D = 3, 3, 4, 2, 40, 8
    rng = np.random.default_rng(14)
    q = rng.standard_normal((B, Tq, H, D))
    kc, vc = rng.standard_normal((B, Tk, Hkv, D)), rng.standard_normal((B, Tk, Hkv, D))
    lens = [40, 17, 4]
    s = 0.4
    for W in (0, 1, 5, 16, 100):
        O, LSE = f(q, kc, vc, lens, s, window=W)
        for b, L in enumerate(lens):
            tq = torch.tensor(q[b:b + 1]).transpose(1, 2)
            tk, tv = (torch.tensor(x[b:b + 1, :L]).transpose(1, 2) for x in (kc, vc))
            pos = torch.arange(L - Tq, L)[:, None]
            j = torch.arange(L)[None, :]
            mask = (j <= pos) & (j >= pos - W)
            ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=s,
                                                                   enable_gqa=True)
            got = O[b:b + 1]
            valid = (pos[:, 0] >= 0).numpy()                # rows before the first key: O = 0 (SDPA gives NaN)
            np.testing.assert_allclose(got[:, valid], ref.transpose(1, 2).numpy()[:, valid], rtol=1e-12,
                                       atol=1e-12)
            logits = s * (tq @ tk.repeat_interleave(H // Hkv, dim=1).transpose(-1, -2))   # [1, H, Tq, L]
            lse_ref = torch.logsumexp(logits.masked_fill(~mask, -np.inf), dim=-1)[0].numpy()
            np.testing.assert_allclose(LSE[b][:, valid], lse_ref[:, valid], rtol=1e-12, atol=1e-12)


def decode_pin_window_limits(f):
    """A window of L - 1 or more is no window; window 0 sees only the query's own key (O = V[p], LSE =
    s q.k_p); Tq = L with a window is the windowed training forward."""
    B, Tq, H, Tk, D = 2, 2, 2, 12, 4
    rng = np.random.default_rng(15)
    q = rng.standard_normal((B, Tq, H, D))
    kc, vc = rng.standard_normal((B, Tk, H, D)), rng.standard_normal((B, Tk, H, D))
    lens = [12, 7]
    s = 0.7
    O0, L0 = f(q, kc, vc, lens, s)
    O1, L1 = f(q, kc, vc, lens, s, window=11)
    np.testing.assert_array_equal(O0, O1)
    np.testing.assert_array_equal(L0, L1)
    Ow, Lw = f(q, kc, vc, lens, s, window=0)
    for b, L in enumerate(lens):
        for i in range(Tq):
            p = L - Tq + i
            np.testing.assert_allclose(Ow[b, i], vc[b, p], rtol=0, atol=1e-15)
            np.testing.assert_allclose(Lw[b, :, i], s * np.einsum("hd,hd->h", q[b, i], kc[b, p]), rtol=1e-13)
    T = 9
    qq, kk, vv = (rng.standard_normal((1, T, H, D)) for _ in range(3))
    Od, Ld = f(qq, kk, vv, [T], s, window=3)
    Of, Lf = attn_ref.attention_forward(qq, kk, vv, s, window=3)
    np.testing.assert_allclose(Od, Of, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(Ld, Lf, rtol=1e-13, atol=1e-13)


DECODE_PINS = [decode_pin_whole_sequence, decode_pin_torch, decode_pin_closed_forms, decode_pin_window_torch,
               decode_pin_window_limits]


@pytest.mark.parametrize("pin", DECODE_PINS)
def test_decode_pins(pin):
    pin(attn_ref.decode_forward)


def _decode_mutant(kind):
    """A copy of the decode oracle with one plausible mistake planted."""
    def f(q, k_cache, v_cache, cache_seqlens, scale, window=None):
        q, kc, vc = (np.asarray(x, dtype=np.float64) for x in (q, k_cache, v_cache))
        if kind == "window_ignored":
            window = None
        B, Tq, H, D = q.shape
        Hkv = kc.shape[2]
        G = H // Hkv
        O, LSE = np.zeros((B, Tq, H, D)), np.full((B, H, Tq), -np.inf)
        for b in range(B):
            L = kc.shape[1] if kind == "lengths_ignored" else int(cache_seqlens[b])
            for h in range(H):
                hk = h % Hkv if kind == "kv_head_modulo" else h // G
                k, v = kc[b, :L, hk], vc[b, :L, hk]
                for i in range(Tq):
                    last = {"top_left_mask": i, "last_key_off_by_one": L - Tq + i - 1}.get(kind, L - Tq + i)
                    if last < 0:
                        continue
                    first = 0
                    if window is not None:
                        first = {"window_one_short": last - window + 1,
                                 "window_from_query_index": i - window}.get(kind, last - window)
                        first = max(0, first)
                    if first > last:
                        continue
                    sc = scale * (k[first: last + 1] @ q[b, i, h])
                    m = sc.max()
                    e = np.exp(sc - m)
                    O[b, i, h] = (e @ v[first: last + 1]) / e.sum()
                    LSE[b, h, i] = m + (np.log2(e.sum()) if kind == "lse_log2" else np.log(e.sum()))
        return O, LSE
    return f


DECODE_MUTANTS = ["lengths_ignored", "kv_head_modulo", "top_left_mask", "last_key_off_by_one", "lse_log2",
                  "window_ignored", "window_one_short", "window_from_query_index"]


def test_decode_mutant_control_passes():
    for pin in DECODE_PINS:
        pin(_decode_mutant("none"))


@pytest.mark.parametrize("kind", DECODE_MUTANTS)
def test_decode_pins_catch_planted_mistake(kind):
    caught = []
    for pin in DECODE_PINS:
        try:
            pin(_decode_mutant(kind))
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no decode pin caught the planted mistake {kind!r}"


# ---------------------------------------------------------------------------------------------------------
# QK normalisation + rotary embedding (the prologue before attention).

def _complex_rotation(xn, pos, base, pairing):
    """The rotary embedding as complex multiplication: the pair (a, b) is a + ib, turned by e^(i p theta_k)."""
    D = xn.shape[-1]
    a, b = (xn[..., 0::2], xn[..., 1::2]) if pairing == "interleaved" else (xn[..., :D // 2], xn[..., D // 2:])
    theta = base ** (-2.0 * np.arange(D // 2) / D)
    z = (a + 1j * b) * np.exp(1j * pos[..., None, None] * theta)
    out = np.empty_like(xn)
    if pairing == "interleaved":
        out[..., 0::2], out[..., 1::2] = z.real, z.imag
    else:
        out[..., :D // 2], out[..., D // 2:] = z.real, z.imag
    return out


def rope_pin_rotation(f, pairing):
    """RMS 1 per head vector (eps = 0); position 0 is the plain normalisation; the rotation equals the complex
    product with e^(i p base^(-2i/D)) (numpy's complex exponential), also with per-sequence offsets."""
    B, T, H, D = 2, 12, 2, 16
    rng = np.random.default_rng(21)
    x = rng.standard_normal((B, T, H, D)) * 3.0
    y = f(x, base=100.0, eps=0.0, pairing=pairing)
    np.testing.assert_allclose(np.sqrt((y * y).mean(axis=-1)), 1.0, rtol=1e-13)
    xn = x / np.sqrt((x * x).mean(axis=-1, keepdims=True))
    np.testing.assert_allclose(y[:, 0], xn[:, 0], rtol=0, atol=1e-14)
    pos = np.broadcast_to(np.arange(T, dtype=np.float64), (B, T))
    np.testing.assert_allclose(y, _complex_rotation(xn, pos, 100.0, pairing), rtol=0, atol=1e-12)
    offs = np.array([5, 40])
    np.testing.assert_allclose(f(x, base=100.0, eps=0.0, offsets=offs, pairing=pairing),
                               _complex_rotation(xn, offs[:, None] + np.arange(T), 100.0, pairing), rtol=0, atol=1e-12)
    np.testing.assert_allclose(f(x[:, 5:], base=100.0, eps=0.0, offsets=5, pairing=pairing), y[:, 5:],
                               rtol=0, atol=1e-12)


def rope_pin_relative_and_eps(f, pairing):
    """q.k after the embedding depends only on the position difference (what rotary embeddings are for); eps
    enters under the square root: with x = 1 everywhere the output RMS is exactly 1 / sqrt(1 + eps)."""
    rng = np.random.default_rng(22)
    T, D = 12, 16
    qv, kv = rng.standard_normal(D), rng.standard_normal(D)
    yq = f(np.broadcast_to(qv, (1, T, 1, D)), base=100.0, pairing=pairing)
    yk = f(np.broadcast_to(kv, (1, T, 1, D)), base=100.0, pairing=pairing)
    dots = [(yq[0, t, 0] * yk[0, t - 3, 0]).sum() for t in range(3, T)]
    np.testing.assert_allclose(dots, dots[0], rtol=1e-12)
    y1 = f(np.ones((1, 4, 1, D)), base=100.0, eps=0.25, pairing=pairing)
    np.testing.assert_allclose(np.sqrt((y1 * y1).mean(axis=-1)), 1.0 / np.sqrt(1.25), rtol=1e-13)


def rope_pin_backward(f, fb, pairing):
    """Central differences of sum(dy * f(x)) in float64, element by element, with per-sequence offsets; with
    eps = 0 the gradient is orthogonal to x (the normalisation is scale-invariant)."""
    rng = np.random.default_rng(8)
    B, T, H, D = 2, 3, 2, 8
    x = rng.standard_normal((B, T, H, D))
    dy = rng.standard_normal((B, T, H, D))
    kw = dict(base=30.0, eps=1e-3, offsets=np.array([0, 7]), pairing=pairing)
    dx = fb(x, dy, **kw)
    num = np.empty_like(x)
    h = 1e-6
    for idx in np.ndindex(x.shape):
        xp, xm = x.copy(), x.copy()
        xp[idx] += h
        xm[idx] -= h
        num[idx] = ((f(xp, **kw) - f(xm, **kw)) * dy).sum() / (2 * h)
    np.testing.assert_allclose(dx, num, rtol=1e-6, atol=1e-8)
    dx0 = fb(x, dy, base=30.0, eps=0.0, pairing=pairing)
    np.testing.assert_allclose((dx0 * x).sum(axis=-1), 0.0, atol=1e-12)


def run_rope_pins(f, fb):
    for pairing in ("interleaved", "half"):
        rope_pin_rotation(f, pairing)
        rope_pin_relative_and_eps(f, pairing)
        rope_pin_backward(f, fb, pairing)


def test_qk_norm_rope_pins():
    run_rope_pins(attn_ref.qk_norm_rope, attn_ref.qk_norm_rope_backward)


def test_rope_pairings_differ_and_match_by_permutation():
    """The two pairings are the same rotation after permuting the dimensions (i, i + D/2) -> (2i, 2i+1)."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((1, 9, 3, 16))
    perm = np.empty(16, dtype=int)
    perm[0::2], perm[1::2] = np.arange(8), np.arange(8, 16)     # interleaved slot j holds half-layout dim perm[j]
    yi = attn_ref.qk_norm_rope(x[..., perm], base=50.0, pairing="interleaved")
    yh = attn_ref.qk_norm_rope(x, base=50.0, pairing="half")
    np.testing.assert_allclose(yi, yh[..., perm], rtol=0, atol=1e-13)
    assert np.abs(attn_ref.qk_norm_rope(x, base=50.0, pairing="interleaved") - yh).max() > 0.1


def _rope_mutant(kind):
    """A copy of the prologue's forward and backward with one plausible mistake planted."""
    def pairs(y, pairing):
        D = y.shape[-1]
        return (y[..., 0::2], y[..., 1::2]) if pairing == "interleaved" else (y[..., :D // 2], y[..., D // 2:])

    def unpairs(a, b, pairing):
        if pairing == "interleaved":
            out = np.empty(a.shape[:-1] + (2 * a.shape[-1],))
            out[..., 0::2], out[..., 1::2] = a, b
            return out
        return np.concatenate([a, b], axis=-1)

    def angles(x, base, offsets):
        B, T, _, D = x.shape
        off = np.broadcast_to(np.asarray(offsets, dtype=np.float64), (B,))
        pos = off[:, None] + np.arange(T)
        if kind == "positions_ignore_offset":
            pos = np.broadcast_to(np.arange(T, dtype=np.float64), (B, T))
        expo = (-1.0 if kind == "freq_exponent_i_over_d" else -2.0) * np.arange(D // 2) / D
        return (pos[:, :, None] * base ** expo)[:, :, None, :]

    def rms(x, eps):
        ms = (x * x).sum(axis=-1, keepdims=True) if kind == "sum_not_mean" else (x * x).mean(axis=-1, keepdims=True)
        return 1.0 / (np.sqrt(ms) + eps) if kind == "eps_outside_sqrt" else 1.0 / np.sqrt(ms + eps)

    def f(x, base=10000.0, eps=1e-6, offsets=0, pairing="interleaved"):
        x = np.asarray(x, dtype=np.float64)
        y = x * rms(x, eps)
        ang = angles(x, base, offsets)
        c, s = np.cos(ang), np.sin(ang)
        if kind == "rotate_backwards":
            s = -s
        a, b = pairs(y, pairing)
        return unpairs(a * c - b * s, a * s + b * c, pairing)

    def fb(x, dy, base=10000.0, eps=1e-6, offsets=0, pairing="interleaved"):
        x, dy = np.asarray(x, dtype=np.float64), np.asarray(dy, dtype=np.float64)
        r = rms(x, eps)
        y = x * r
        ang = angles(x, base, offsets)
        c, s = np.cos(ang), np.sin(ang)
        if kind == "bwd_rotates_forward":
            s = -s
        a, b = pairs(dy, pairing)
        g = unpairs(a * c + b * s, -a * s + b * c, pairing)
        if kind == "bwd_drops_projection":
            return r * g
        return r * (g - y * (g * y).mean(axis=-1, keepdims=True))

    return f, fb


ROPE_MUTANTS = ["positions_ignore_offset", "freq_exponent_i_over_d", "sum_not_mean", "eps_outside_sqrt",
                "rotate_backwards", "bwd_rotates_forward", "bwd_drops_projection"]


def test_rope_mutant_control_passes():
    run_rope_pins(*_rope_mutant("none"))


@pytest.mark.parametrize("kind", ROPE_MUTANTS)
def test_rope_pins_catch_planted_mistake(kind):
    with pytest.raises(AssertionError):
        run_rope_pins(*_rope_mutant(kind))


# ---------------------------------------------------------------------------------------------------------
# Mutation test: plant plausible mistakes in a copy of the oracle and require that some pin fails.

def _mutant(kind):
    def fwd(q, k, v, s):
        T = q.shape[0]
        S = s * (q @ (k if kind == "no_transpose_qk" else k).T)
        off = -1 if kind == "mask_excludes_diagonal" else 0
        mask = np.tril(np.ones((T, T), dtype=bool), k=off)
        if kind == "mask_excludes_diagonal":
            mask[0, 0] = True
        if kind == "no_mask":
            mask[:] = True
        S = np.where(mask, S, -np.inf)
        m = S.max(axis=1, keepdims=True)
        E = np.exp(S - m)
        l = E.sum(axis=1, keepdims=True)
        P = E / l
        O = (P.T if kind == "transposed_pv" else P) @ v
        lse = (m + (np.log2(l) if kind == "lse_log2" else np.log(l)))[:, 0]
        return O, lse, P

    def bwd(q, k, v, do, s):
        O, _, P = fwd(q, k, v, s)
        dV = (P @ do) if kind == "dv_not_transposed" else P.T @ do
        dP = do @ v.T
        delta = (do * O).sum(axis=1)
        dS = P * (dP + delta[:, None]) if kind == "delta_sign" else P * (dP - delta[:, None])
        if kind == "dropped_delta":
            dS = P * dP
        dQ = (1.0 if kind == "dq_no_scale" else s) * (dS @ k)
        dK = (1.0 if kind == "dk_no_scale" else s) * (dS.T @ q)
        if kind == "dk_uses_k":
            dK = s * (dS.T @ k)
        return dQ, dK, dV, delta

    return fwd, bwd


MUTANTS = ["mask_excludes_diagonal", "no_mask", "transposed_pv", "lse_log2", "dv_not_transposed", "delta_sign",
           "dropped_delta", "dq_no_scale", "dk_no_scale", "dk_uses_k"]


def test_mutant_control_passes():
    """The mutant factory without a mutation reproduces the oracle, so a failure below is the planted bug."""
    for pin in ALL_PINS:
        pin(_mutant("none"))


@pytest.mark.parametrize("kind", MUTANTS)
def test_pins_catch_planted_mistake(kind):
    impl = _mutant(kind)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(impl)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {kind!r}"
