"""Pins for the double-precision oracle (CPU only).

The oracle computes the WKV operator with the O(T) recurrences the pages state.
Nothing here re-types those recurrences: each test checks the oracle against
something fixed independently of it -- the brute-force O(T^2) pair sums
(tests/brute.py), hand-derived fixtures (tests/golden), plain matmul
reductions, closed forms, symmetries, Euler identities and finite differences.
"""
import json
import math
import os

import numpy as np
import pytest

from tests import brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _wkv6_case(B, T, H, N, seed, wlo=-3.0, whi=-0.05):
    g = _rng(seed)
    C = H * N
    r = g.normal(0, 0.7, (B, T, C))
    k = g.normal(0, 0.7, (B, T, C))
    v = g.normal(0, 0.7, (B, T, C))
    w = -np.exp(g.uniform(wlo, whi, (B, T, C)))
    u = g.normal(0, 0.7, C)
    return r, k, v, w, u


def _flip(*arrs):
    return [a[:, ::-1].copy() for a in arrs]


# ---------------------------------------------------------------- hand-derived fixtures

def test_golden_wkv6_forward(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "wkv6_fwd_t4n2.json")))
    arr = lambda key: np.array(g[key], dtype=np.float64)[None]
    r, k, v = arr("r"), arr("k"), arr("v")
    w = np.log(arr("decay"))
    u = np.array(g["u"], dtype=np.float64)
    y = oracle_mod.wkv6_fwd(r, k, v, w, u, H=1, bidirectional=False)
    np.testing.assert_allclose(y[0], g["y_causal"], rtol=0, atol=1e-12)
    yb = oracle_mod.wkv6_fwd(r, k, v, w, u, H=1, bidirectional=True)
    np.testing.assert_allclose(yb[0], g["y_bidir"], rtol=0, atol=1e-12)


@pytest.mark.parametrize("mode", ["causal", "bidir"])
def test_golden_wkv6_backward(oracle_mod, mode):
    g = json.load(open(os.path.join(GOLDEN, "wkv6_bwd_t3n1.json")))
    col = lambda key: np.array(g[key], dtype=np.float64).reshape(1, -1, 1)
    r, k, v, dy = col("r"), col("k"), col("v"), col("dy")
    w = np.log(col("decay"))
    u = np.array([g["u"]], dtype=np.float64)
    bid = mode == "bidir"
    y = oracle_mod.wkv6_fwd(r, k, v, w, u, H=1, bidirectional=bid)
    np.testing.assert_allclose(y.ravel(), g[f"y_{mode}"], atol=1e-12)
    dr, dk, dv, dw, du = oracle_mod.wkv6_bwd(r, k, v, w, u, dy, H=1, bidirectional=bid)
    for name, got in (("dr", dr), ("dk", dk), ("dv", dv), ("dw", dw)):
        np.testing.assert_allclose(got.ravel(), g[f"{name}_{mode}"], atol=1e-12, err_msg=name)
    assert abs(du[0] - g[f"du_{mode}"]) < 1e-12


def test_golden_wkv4_forward(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "wkv4_fwd_t3c1.json")))
    k = np.array(g["k"], dtype=np.float64).reshape(1, -1, 1)
    v = np.array(g["v"], dtype=np.float64).reshape(1, -1, 1)
    y = oracle_mod.wkv4_fwd(k, v, np.array([g["w"]]), np.array([g["u"]]))
    np.testing.assert_allclose(y.ravel(), g["y"], rtol=1e-14, atol=1e-14)


# ---------------------------------------------------------------- RWKV-6 forward

@pytest.mark.parametrize("B,T,H,N", [(1, 1, 1, 4), (2, 2, 1, 4), (1, 3, 2, 8), (2, 7, 2, 4),
                                     (1, 33, 1, 8), (1, 7, 1, 64)])
@pytest.mark.parametrize("bidir", [False, True])
def test_wkv6_recurrence_matches_pair_sums(oracle_mod, B, T, H, N, bidir):
    r, k, v, w, u = _wkv6_case(B, T, H, N, seed=T * 100 + N + bidir)
    y = oracle_mod.wkv6_fwd(r, k, v, w, u, H=H, bidirectional=bidir)
    yb = brute.wkv6(r, k, v, w, u, H, past=True, future=bidir, bonus=True)
    assert np.max(np.abs(y - yb)) <= 1e-12 * max(1.0, np.max(np.abs(yb)))


def test_wkv6_no_decay_is_masked_matmul(oracle_mod):
    """ew = 0 (decay 1) and u = 1: causal = tril(R K^T) V, bidirectional = (R K^T) V."""
    T, N = 9, 8
    g = _rng(3)
    R, K, V = (g.normal(size=(T, N)) for _ in range(3))
    w = np.zeros((1, T, N))
    u = np.ones(N)
    yc = oracle_mod.wkv6_fwd(R[None], K[None], V[None], w, u, H=1)[0]
    np.testing.assert_allclose(yc, np.tril(R @ K.T) @ V, rtol=1e-12, atol=1e-12)
    yb = oracle_mod.wkv6_fwd(R[None], K[None], V[None], w, u, H=1, bidirectional=True)[0]
    np.testing.assert_allclose(yb, (R @ K.T) @ V, rtol=1e-12, atol=1e-12)


def test_wkv6_full_decay_closed_form(oracle_mod):
    """decay 0 (ew = -inf): only the previous token survives: y_t = r_t.(k_{t-1}^T v_{t-1} + diag(u) k_t^T v_t)."""
    r, k, v, _, u = _wkv6_case(1, 6, 1, 4, seed=5)
    w = np.full(r.shape, -np.inf)
    y = oracle_mod.wkv6_fwd(r, k, v, w, u, H=1)[0]
    R, K, V = r[0], k[0], v[0]
    for t in range(6):
        exp = (R[t] * u * K[t]).sum() * V[t]
        if t > 0:
            exp = exp + (R[t] * K[t - 1]).sum() * V[t - 1]
        np.testing.assert_allclose(y[t], exp, rtol=1e-13, atol=1e-13)


def test_wkv6_single_token_closed_form(oracle_mod):
    r, k, v, w, u = _wkv6_case(2, 1, 3, 4, seed=6)
    for bid in (False, True):
        y = oracle_mod.wkv6_fwd(r, k, v, w, u, H=3, bidirectional=bid)
        for h in range(3):
            sl = slice(4 * h, 4 * h + 4)
            c = (r[:, 0, sl] * u[sl] * k[:, 0, sl]).sum(-1, keepdims=True)
            np.testing.assert_allclose(y[:, 0, sl], c * v[:, 0, sl], rtol=1e-13, atol=1e-13)


def test_wkv6_bidir_is_causal_plus_anticausal_minus_bonus(oracle_mod):
    B, T, H, N = 2, 17, 2, 8
    r, k, v, w, u = _wkv6_case(B, T, H, N, seed=7)
    yc = oracle_mod.wkv6_fwd(r, k, v, w, u, H=H)
    ya = oracle_mod.wkv6_fwd(*_flip(r, k, v, w), u, H=H)[:, ::-1]
    bonus = np.zeros_like(yc)
    for h in range(H):
        sl = slice(h * N, (h + 1) * N)
        bonus[..., sl] = (r[..., sl] * u[sl] * k[..., sl]).sum(-1, keepdims=True) * v[..., sl]
    yb = oracle_mod.wkv6_fwd(r, k, v, w, u, H=H, bidirectional=True)
    np.testing.assert_allclose(yb, yc + ya - bonus, rtol=1e-11, atol=1e-11)


def test_wkv6_bidir_reversal_symmetry(oracle_mod):
    r, k, v, w, u = _wkv6_case(2, 13, 2, 8, seed=8)
    yb = oracle_mod.wkv6_fwd(r, k, v, w, u, H=2, bidirectional=True)
    yf = oracle_mod.wkv6_fwd(*_flip(r, k, v, w), u, H=2, bidirectional=True)
    np.testing.assert_allclose(yf[:, ::-1], yb, rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("bidir", [False, True])
def test_wkv6_linear_in_r_and_v(oracle_mod, bidir):
    r, k, v, w, u = _wkv6_case(1, 11, 2, 4, seed=9)
    g = _rng(10)
    r2, v2 = g.normal(size=r.shape), g.normal(size=v.shape)
    f = lambda rr, vv: oracle_mod.wkv6_fwd(rr, k, vv, w, u, H=2, bidirectional=bidir)
    np.testing.assert_allclose(f(2.0 * r - 3.0 * r2, v), 2.0 * f(r, v) - 3.0 * f(r2, v), rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(f(r, 0.5 * v + v2), 0.5 * f(r, v) + f(r, v2), rtol=1e-11, atol=1e-11)


def test_wkv6_heads_and_batches_are_independent(oracle_mod):
    B, T, H, N = 2, 9, 3, 4
    r, k, v, w, u = _wkv6_case(B, T, H, N, seed=11)
    y = oracle_mod.wkv6_fwd(r, k, v, w, u, H=H, bidirectional=True)
    for b in range(B):
        for h in range(H):
            sl = slice(h * N, (h + 1) * N)
            ys = oracle_mod.wkv6_fwd(r[b:b + 1, :, sl], k[b:b + 1, :, sl], v[b:b + 1, :, sl],
                                     w[b:b + 1, :, sl], u[sl], H=1, bidirectional=True)
            np.testing.assert_array_equal(ys[0], y[b, :, sl])


def test_wkv6_decay_indexing(oracle_mod):
    """d_0 and d_{T-1} never reach a causal output; d_0 and d_{T-1} never reach an
    anti-causal one either (the state is read before the step's decay applies)."""
    r, k, v, w, u = _wkv6_case(1, 6, 1, 4, seed=12)
    for bid in (False, True):
        y = oracle_mod.wkv6_fwd(r, k, v, w, u, H=1, bidirectional=bid)
        w2 = w.copy()
        w2[:, 0] -= 1.3
        w2[:, -1] -= 0.7
        np.testing.assert_array_equal(oracle_mod.wkv6_fwd(r, k, v, w2, u, H=1, bidirectional=bid), y)
        w3 = w.copy()
        w3[:, 2] -= 0.5
        assert np.max(np.abs(oracle_mod.wkv6_fwd(r, k, v, w3, u, H=1, bidirectional=bid) - y)) > 1e-3


# ---------------------------------------------------------------- RWKV-6 backward

def _loss(oracle_mod, r, k, v, w, u, dy, H, bid):
    return float(np.sum(dy * oracle_mod.wkv6_fwd(r, k, v, w, u, H=H, bidirectional=bid)))


@pytest.mark.parametrize("bidir", [False, True])
def test_wkv6_backward_finite_differences(oracle_mod, bidir):
    B, T, H, N = 1, 6, 2, 3
    r, k, v, w, u = _wkv6_case(B, T, H, N, seed=20 + bidir, wlo=-1.5, whi=0.0)
    dy = _rng(21).normal(size=r.shape)
    grads = oracle_mod.wkv6_bwd(r, k, v, w, u, dy, H=H, bidirectional=bidir)
    eps = 1e-6
    for name, arr, g in zip(("r", "k", "v", "w", "u"), (r, k, v, w, u), grads):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            args = {"r": r, "k": k, "v": v, "w": w, "u": u}
            hi = arr.copy(); hi[idx] += eps
            lo = arr.copy(); lo[idx] -= eps
            args[name] = hi
            fp = _loss(oracle_mod, args["r"], args["k"], args["v"], args["w"], args["u"], dy, H, bidir)
            args[name] = lo
            fm = _loss(oracle_mod, args["r"], args["k"], args["v"], args["w"], args["u"], dy, H, bidir)
            num[idx] = (fp - fm) / (2 * eps)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-7, err_msg=name)


@pytest.mark.parametrize("bidir", [False, True])
@pytest.mark.parametrize("T,N", [(1, 4), (2, 4), (9, 4), (12, 8)])
def test_wkv6_backward_matches_pair_form(oracle_mod, bidir, T, N):
    r, k, v, w, u = _wkv6_case(1, T, 1, N, seed=30 + T + bidir)
    dy = _rng(31).normal(size=r.shape)
    got = oracle_mod.wkv6_bwd(r, k, v, w, u, dy, H=1, bidirectional=bidir)
    exp = brute.wkv6_head_grads(r[0], k[0], v[0], w[0], u, dy[0], past=True, future=bidir)
    for name, g, e in zip(("dr", "dk", "dv", "dw"), got[:4], exp[:4]):
        np.testing.assert_allclose(g[0], e, rtol=1e-11, atol=1e-11, err_msg=name)
    np.testing.assert_allclose(got[4], exp[4], rtol=1e-11, atol=1e-11, err_msg="du")


@pytest.mark.parametrize("bidir", [False, True])
def test_wkv6_backward_euler_identities(oracle_mod, bidir):
    """y is degree-1 homogeneous in r, in k and in v separately, and the bonus is linear in u."""
    B, T, H, N = 2, 15, 2, 8
    r, k, v, w, u = _wkv6_case(B, T, H, N, seed=40 + bidir)
    dy = _rng(41).normal(size=r.shape)
    y = oracle_mod.wkv6_fwd(r, k, v, w, u, H=H, bidirectional=bidir)
    dr, dk, dv, dw, du = oracle_mod.wkv6_bwd(r, k, v, w, u, dy, H=H, bidirectional=bidir)
    ref = float(np.sum(dy * y))
    for g, x in ((dr, r), (dk, k), (dv, v)):
        assert abs(float(np.sum(g * x)) - ref) <= 1e-10 * max(1.0, abs(ref))
    bonus_part = ref - float(np.sum(dy * oracle_mod.wkv6_fwd(r, k, v, w, np.zeros_like(u), H=H, bidirectional=bidir)))
    assert abs(float(du @ u) - bonus_part) <= 1e-10 * max(1.0, abs(bonus_part))


@pytest.mark.parametrize("bidir", [False, True])
def test_wkv6_backward_dw_vanishes_at_ends(oracle_mod, bidir):
    r, k, v, w, u = _wkv6_case(2, 10, 2, 4, seed=50)
    dy = _rng(51).normal(size=r.shape)
    dw = oracle_mod.wkv6_bwd(r, k, v, w, u, dy, H=2, bidirectional=bidir)[3]
    assert np.all(dw[:, 0] == 0.0) and np.all(dw[:, -1] == 0.0)
    assert np.max(np.abs(dw[:, 1:-1])) > 1e-3


# ---------------------------------------------------------------- RWKV-4

def _wkv4_case(B, T, C, seed, kstd=1.0):
    g = _rng(seed)
    k = g.normal(0, kstd, (B, T, C))
    v = g.normal(0, 1, (B, T, C))
    w = np.exp(g.uniform(-3, 1, C))
    u = g.normal(0, 0.5, C)
    return k, v, w, u


# ---------------------------------------------------------------- state carried across calls

@pytest.mark.parametrize("B,T,H,N", [(1, 1, 1, 4), (2, 3, 1, 4), (1, 7, 2, 8), (1, 33, 1, 8), (1, 5, 1, 64)])
def test_wkv6_state_matches_pair_form(oracle_mod, B, T, H, N):
    """y and the final state from an initial state s0 equal the pair sums with s0 decayed explicitly."""
    r, k, v, w, u = _wkv6_case(B, T, H, N, seed=700 + 10 * T + N)
    s0 = _rng(7 + T).normal(0, 1.0, (B, H, N, N))
    y, sT = oracle_mod.wkv6_fwd_state(r, k, v, w, u, H, s0)
    for b in range(B):
        for h in range(H):
            sl = slice(h * N, (h + 1) * N)
            yb, sb = brute.wkv6_head_state(r[b, :, sl], k[b, :, sl], v[b, :, sl], w[b, :, sl], u[sl], s0[b, h])
            assert np.max(np.abs(y[b, :, sl] - yb)) <= 1e-12 * max(1.0, np.max(np.abs(yb)))
            assert np.max(np.abs(sT[b, h] - sb)) <= 1e-12 * max(1.0, np.max(np.abs(sb)))


@pytest.mark.parametrize("cut", [0, 1, 13, 28, 29])
def test_wkv6_state_split_equals_whole(oracle_mod, cut):
    """Running tokens [0, cut) and then [cut, T) from the carried state reproduces the whole run."""
    B, T, H, N = 2, 29, 2, 8
    r, k, v, w, u = _wkv6_case(B, T, H, N, seed=901)
    s0 = _rng(902).normal(0, 1.0, (B, H, N, N))
    y, sT = oracle_mod.wkv6_fwd_state(r, k, v, w, u, H, s0)
    a, z = slice(0, cut), slice(cut, T)
    y1, s1 = oracle_mod.wkv6_fwd_state(r[:, a], k[:, a], v[:, a], w[:, a], u, H, s0)
    y2, s2 = oracle_mod.wkv6_fwd_state(r[:, z], k[:, z], v[:, z], w[:, z], u, H, s1)
    tol = 1e-12 * max(1.0, np.max(np.abs(y)))
    assert np.max(np.abs(np.concatenate([y1, y2], axis=1) - y)) <= tol
    assert np.max(np.abs(s2 - sT)) <= 1e-12 * max(1.0, np.max(np.abs(sT)))


def test_wkv6_state_zero_is_the_plain_forward(oracle_mod):
    B, T, H, N = 2, 11, 2, 4
    r, k, v, w, u = _wkv6_case(B, T, H, N, seed=911)
    y_plain = oracle_mod.wkv6_fwd(r, k, v, w, u, H=H)
    y_none, s_none = oracle_mod.wkv6_fwd_state(r, k, v, w, u, H, None)
    y_zero, s_zero = oracle_mod.wkv6_fwd_state(r, k, v, w, u, H, np.zeros((B, H, N, N)))
    assert np.array_equal(y_none, y_plain) and np.array_equal(y_zero, y_plain)
    assert np.array_equal(s_none, s_zero)
    # no tokens: the state passes through unchanged
    s0 = _rng(912).normal(0, 1.0, (B, H, N, N))
    e = slice(0, 0)
    y0, s_out = oracle_mod.wkv6_fwd_state(r[:, e], k[:, e], v[:, e], w[:, e], u, H, s0)
    assert y0.shape == (B, 0, H * N) and np.array_equal(s_out, s0)


@pytest.mark.parametrize("B,T,C", [(1, 1, 3), (2, 5, 3), (1, 40, 4)])
def test_wkv4_recurrence_matches_ratio_of_sums(oracle_mod, B, T, C):
    k, v, w, u = _wkv4_case(B, T, C, seed=60 + T)
    y = oracle_mod.wkv4_fwd(k, v, w, u)
    np.testing.assert_allclose(y, brute.wkv4(k, v, w, u), rtol=1e-12, atol=1e-12)


def test_wkv4_closed_forms(oracle_mod):
    k, v, w, u = _wkv4_case(2, 12, 5, seed=61)
    y = oracle_mod.wkv4_fwd(k, v, w, u)
    np.testing.assert_allclose(y[:, 0], v[:, 0], rtol=1e-14)          # first token: y_0 = v_0
    yc = oracle_mod.wkv4_fwd(k, np.full_like(v, 2.5), w, u)           # constant v: convex combination
    np.testing.assert_allclose(yc, 2.5, rtol=1e-13)
    for t in range(1, 12):                                            # bounds of a convex combination
        lo, hi = v[:, :t + 1].min(1), v[:, :t + 1].max(1)
        assert np.all(y[:, t] >= lo - 1e-12) and np.all(y[:, t] <= hi + 1e-12)


def test_wkv4_geometric_closed_form(oracle_mod):
    """k = 0, v_s = 1 for s < t and v_t = 0: y_t = b / (b + e^u), b = (1 - e^{-t w}) / (1 - e^{-w})."""
    T, C = 9, 3
    w = np.array([0.2, 1.0, 2.5])
    u = np.array([-0.3, 0.0, 0.8])
    for t in range(1, T):
        v = np.ones((1, T, C))
        v[:, t] = 0.0
        y = oracle_mod.wkv4_fwd(np.zeros((1, T, C)), v, w, u)
        b = (1 - np.exp(-t * w)) / (1 - np.exp(-w))
        np.testing.assert_allclose(y[0, t], b / (b + np.exp(u)), rtol=1e-13)


def test_wkv4_large_keys_stay_finite(oracle_mod):
    """k ~ N(0, 30^2): exp(k) overflows float32; the log-space state keeps the ratio exact."""
    k, v, w, u = _wkv4_case(1, 60, 3, seed=62, kstd=30.0)
    y = oracle_mod.wkv4_fwd(k, v, w, u)
    assert np.all(np.isfinite(y))
    np.testing.assert_allclose(y, brute.wkv4(k, v, w, u), rtol=1e-11, atol=1e-11)
    k2 = k.copy(); k2 += 500.0                                        # a common shift of k, u cancels
    np.testing.assert_allclose(oracle_mod.wkv4_fwd(k2, v, w, u), y, rtol=1e-9, atol=1e-9)


# ---------------------------------------------------------------- RWKV-4 backward

def _wkv4_loss(oracle_mod, k, v, w, u, dy):
    return float(np.sum(dy * oracle_mod.wkv4_fwd(k, v, w, u)))


@pytest.mark.parametrize("B,T,C", [(1, 1, 2), (2, 5, 3), (1, 9, 2)])
def test_wkv4_backward_finite_differences(oracle_mod, B, T, C):
    """Central differences of the forward oracle (L = sum dy * y) reproduce every gradient."""
    k, v, w, u = _wkv4_case(B, T, C, seed=500 + T)
    dy = _rng(501 + T).normal(0, 1, (B, T, C))
    dk, dv, dw, du = oracle_mod.wkv4_bwd(k, v, w, u, dy)
    h = 1e-6

    def fd(arr, idx):
        a1, a2 = arr.copy(), arr.copy()
        a1[idx] += h
        a2[idx] -= h
        return a1, a2

    for name, grad, pos in (("dk", dk, 0), ("dv", dv, 1)):
        for idx in np.ndindex(grad.shape):
            args1, args2 = [k, v, w, u], [k, v, w, u]
            args1[pos], args2[pos] = fd([k, v][pos], idx)
            num = (_wkv4_loss(oracle_mod, *args1, dy) - _wkv4_loss(oracle_mod, *args2, dy)) / (2 * h)
            assert abs(num - grad[idx]) <= 1e-6 * max(1.0, abs(num)), (name, idx, num, grad[idx])
    for name, grad, pos in (("dw", dw, 2), ("du", du, 3)):
        for c in range(C):
            args1, args2 = [k, v, w, u], [k, v, w, u]
            args1[pos], args2[pos] = fd([w, u][pos - 2], (c,))
            num = (_wkv4_loss(oracle_mod, *args1, dy) - _wkv4_loss(oracle_mod, *args2, dy)) / (2 * h)
            assert abs(num - grad[c]) <= 1e-6 * max(1.0, abs(num)), (name, c, num, grad[c])


def test_wkv4_backward_invariants(oracle_mod):
    """y is unchanged by a common shift of all k (so dk sums to 0 per sequence) and is
    homogeneous of degree 1 in v (so <v, dv> = <dy, y> per sequence); T = 1 gives y = v."""
    B, T, C = 2, 17, 4
    k, v, w, u = _wkv4_case(B, T, C, seed=520)
    dy = _rng(521).normal(0, 1, (B, T, C))
    dk, dv, dw, du = oracle_mod.wkv4_bwd(k, v, w, u, dy)
    y = oracle_mod.wkv4_fwd(k, v, w, u)
    assert np.max(np.abs(dk.sum(axis=1))) <= 1e-12 * max(1.0, np.max(np.abs(dk)))
    np.testing.assert_allclose(np.sum(v * dv, axis=1), np.sum(dy * y, axis=1), rtol=1e-12, atol=1e-12)
    k1, v1, w1, u1 = _wkv4_case(2, 1, 3, seed=522)
    dy1 = _rng(523).normal(0, 1, (2, 1, 3))
    dk1, dv1, dw1, du1 = oracle_mod.wkv4_bwd(k1, v1, w1, u1, dy1)
    assert np.allclose(dv1, dy1, rtol=0, atol=1e-15) and not np.any(dk1) and not np.any(dw1) and not np.any(du1)


def test_wkv4_backward_large_keys_stay_finite(oracle_mod):
    """k ~ N(0, 30^2): every exponent is shifted by the step's largest one, so nothing overflows;
    the invariants still hold."""
    k, v, w, u = _wkv4_case(1, 40, 3, seed=530, kstd=30.0)
    dy = _rng(531).normal(0, 1, k.shape)
    dk, dv, dw, du = oracle_mod.wkv4_bwd(k, v, w, u, dy)
    for g in (dk, dv, dw, du):
        assert np.all(np.isfinite(g))
    y = oracle_mod.wkv4_fwd(k, v, w, u)
    np.testing.assert_allclose(np.sum(v * dv, axis=1), np.sum(dy * y, axis=1), rtol=1e-10, atol=1e-10)


# ---------------------------------------------------------------- planted mistakes are caught

def test_pins_catch_a_planted_decay_index_error():
    """A plausible mistake (applying d_t before reading y_t) must fail the pair-sum pin."""
    r, k, v, w, u = _wkv6_case(1, 8, 1, 4, seed=70)
    R, K, V, W = r[0], k[0], v[0], w[0]
    S = np.zeros((4, 4))
    y = np.zeros((8, 4))
    for t in range(8):
        S = np.exp(W[t])[:, None] * S           # wrong order: decay first
        y[t] = R[t] @ (S + np.diag(u) @ np.outer(K[t], V[t]))
        S = S + np.outer(K[t], V[t])
    yb = brute.wkv6_head(R, K, V, W, u)
    assert np.max(np.abs(y - yb)) > 1e-3


# ---------------------------------------------------------------- RWKV-5 (static decay)

def _wkv5_case(B, T, H, N, seed, wlo=-3.0, whi=1.0):
    g = _rng(seed)
    C = H * N
    r, k, v = (g.normal(0, 0.7, (B, T, C)) for _ in range(3))
    w = np.exp(g.uniform(wlo, whi, C))            # decay exp(-w) per channel
    u = g.normal(0, 0.7, C)
    return r, k, v, w, u


@pytest.mark.parametrize("B,T,H,N", [(1, 1, 1, 4), (2, 7, 2, 4), (1, 33, 1, 8), (1, 5, 1, 64)])
def test_wkv5_is_wkv6_with_constant_decay(oracle_mod, B, T, H, N):
    """RWKV-5 is the static special case: the brute-force pair sums with ew_t = -w for every t."""
    r, k, v, w, u = _wkv5_case(B, T, H, N, seed=60 + T)
    y = oracle_mod.wkv5_fwd(r, k, v, w, u, H=H)
    yb = brute.wkv6(r, k, v, np.broadcast_to(-w, r.shape).copy(), u, H)
    assert np.max(np.abs(y - yb)) <= 1e-12 * max(1.0, np.max(np.abs(yb)))


def test_wkv5_geometric_closed_form(oracle_mod):
    """One live channel i with k = 1 and v = 1: y_t[j] = r_t[i] ((1 - d^t) / (1 - d) + u_i), d = e^{-w_i}."""
    T, N, i = 12, 4, 2
    r = np.zeros((1, T, N)); r[0, :, i] = _rng(61).normal(size=T)
    k = np.zeros((1, T, N)); k[0, :, i] = 1.0
    v = np.ones((1, T, N))
    w = np.array([0.3, 1.1, 0.45, 2.0]); u = np.array([0.1, -0.2, 0.7, 0.4])
    y = oracle_mod.wkv5_fwd(r, k, v, w, u, H=1)[0]
    d = math.exp(-w[i])
    for t in range(T):
        exp = r[0, t, i] * ((1 - d ** t) / (1 - d) + u[i])
        np.testing.assert_allclose(y[t], np.full(N, exp), rtol=1e-13, atol=1e-13)


def test_wkv5_no_decay_is_masked_matmul(oracle_mod):
    """w = 0 (decay 1), u = 1: y = tril(R K^T) V."""
    T, N = 9, 8
    g = _rng(62)
    R, K, V = (g.normal(size=(T, N)) for _ in range(3))
    y = oracle_mod.wkv5_fwd(R[None], K[None], V[None], np.zeros(N), np.ones(N), H=1)[0]
    np.testing.assert_allclose(y, np.tril(R @ K.T) @ V, rtol=1e-12, atol=1e-12)


def test_wkv5_backward_finite_differences(oracle_mod):
    B, T, H, N = 2, 6, 2, 3
    r, k, v, w, u = _wkv5_case(B, T, H, N, seed=63, wlo=-2.0, whi=0.5)
    dy = _rng(64).normal(size=r.shape)
    grads = oracle_mod.wkv5_bwd(r, k, v, w, u, dy, H=H)
    loss = lambda a: float(np.sum(dy * oracle_mod.wkv5_fwd(a["r"], a["k"], a["v"], a["w"], a["u"], H=H)))
    eps = 1e-6
    for name, arr, g in zip(("r", "k", "v", "w", "u"), (r, k, v, w, u), grads):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            args = {"r": r, "k": k, "v": v, "w": w, "u": u}
            hi = arr.copy(); hi[idx] += eps
            lo = arr.copy(); lo[idx] -= eps
            args[name] = hi
            fp = loss(args)
            args[name] = lo
            fm = loss(args)
            num[idx] = (fp - fm) / (2 * eps)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-7, err_msg=name)


def test_wkv5_backward_matches_summed_wkv6_pair_form(oracle_mod):
    """dr, dk, dv, du equal RWKV-6's at ew = -w; dw[c] is minus the per-token RWKV-6 dw summed over b, t."""
    B, T, H, N = 2, 9, 1, 4
    r, k, v, w, u = _wkv5_case(B, T, H, N, seed=65)
    dy = _rng(66).normal(size=r.shape)
    dr, dk, dv, dw, du = oracle_mod.wkv5_bwd(r, k, v, w, u, dy, H=H)
    ew = np.broadcast_to(-w, r.shape[1:]).copy()
    dw_sum = np.zeros(N); du_sum = np.zeros(N)
    for b in range(B):
        e = brute.wkv6_head_grads(r[b], k[b], v[b], ew, u, dy[b], past=True, future=False)
        for name, got, ref in zip(("dr", "dk", "dv"), (dr[b], dk[b], dv[b]), e[:3]):
            np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-11, err_msg=name)
        dw_sum -= e[3].sum(0)
        du_sum += e[4]
    np.testing.assert_allclose(dw, dw_sum, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(du, du_sum, rtol=1e-11, atol=1e-11)


# ---------------------------------------------------------------- fused prologue / epilogue

def _fused_case(B, T, H, N, seed):
    g = _rng(seed)
    C = H * N
    r, k, v = (g.normal(0, 0.7, (B, T, C)) for _ in range(3))
    ww = g.normal(0, 0.5, (B, T, C))                 # LoRA part of the decay pre-activation
    wb = g.uniform(-4.0, -0.5, C)                    # w_base
    u = g.normal(0, 0.7, C)
    gate = g.normal(0, 1.0, (B, T, C))
    gn_w, gn_b = g.normal(1.0, 0.3, C), g.normal(0, 0.3, C)
    return r, k, v, ww, wb, u, gate, gn_w, gn_b


@pytest.mark.parametrize("bidir", [False, True])
def test_fused_matches_library_group_norm(oracle_mod, bidir):
    """out = torch group_norm(y, H groups, gn_w, gn_b, eps) * g, with y the pinned RWKV-6
    forward at ew = -exp(w_base + ww)."""
    torch = pytest.importorskip("torch")
    B, T, H, N = 2, 11, 3, 8
    r, k, v, ww, wb, u, gate, gn_w, gn_b = _fused_case(B, T, H, N, seed=70 + bidir)
    eps = 1e-3
    out = oracle_mod.wkv6_fwd_fused(r, k, v, ww, wb, u, gate, gn_w, gn_b, eps, H=H, bidirectional=bidir)
    y = oracle_mod.wkv6_fwd(r, k, v, -np.exp(wb + ww), u, H=H, bidirectional=bidir)
    gn = torch.nn.functional.group_norm(torch.from_numpy(y.reshape(B * T, H * N)), H,
                                        torch.from_numpy(gn_w), torch.from_numpy(gn_b), eps).numpy()
    np.testing.assert_allclose(out, gn.reshape(B, T, H * N) * gate, rtol=1e-12, atol=1e-12)


def test_fused_rows_are_normalised_per_head(oracle_mod):
    """Unit affine and gate: every (token, head) row has mean 0 and mean square var / (var + eps)."""
    B, T, H, N = 1, 9, 2, 16
    r, k, v, ww, wb, u, _, _, _ = _fused_case(B, T, H, N, seed=72)
    C = H * N
    out = oracle_mod.wkv6_fwd_fused(r, k, v, ww, wb, u, np.ones((B, T, C)), np.ones(C), np.zeros(C), 1e-14, H=H)
    rows = out.reshape(B * T, H, N)
    assert np.max(np.abs(rows.mean(-1))) <= 1e-12
    np.testing.assert_allclose((rows ** 2).mean(-1), 1.0, rtol=1e-9)


def test_fused_scale_invariance_and_affine_order(oracle_mod):
    """Scaling v by a > 0 scales y and leaves the normalised output unchanged (eps -> 0); the
    affine map acts before the gate: out(gn_w, gn_b, g) = (out(1, 0, 1) * gn_w + gn_b) * g."""
    B, T, H, N = 2, 7, 2, 8
    r, k, v, ww, wb, u, gate, gn_w, gn_b = _fused_case(B, T, H, N, seed=73)
    C = H * N
    one, zero = np.ones(C), np.zeros(C)
    base = oracle_mod.wkv6_fwd_fused(r, k, v, ww, wb, u, np.ones_like(gate), one, zero, 1e-14, H=H)
    scaled = oracle_mod.wkv6_fwd_fused(r, k, 3.5 * v, ww, wb, u, np.ones_like(gate), one, zero, 1e-14, H=H)
    np.testing.assert_allclose(scaled, base, rtol=1e-8, atol=1e-9)
    full = oracle_mod.wkv6_fwd_fused(r, k, v, ww, wb, u, gate, gn_w, gn_b, 1e-14, H=H)
    np.testing.assert_allclose(full, (base * gn_w + gn_b) * gate, rtol=1e-12, atol=1e-12)


def test_fused_prologue_moves_constant_between_base_and_lora(oracle_mod):
    """Only w_base + ww enters the decay: shifting a per-channel constant from one to the other
    changes nothing, and a different sum changes the output."""
    B, T, H, N = 1, 8, 2, 4
    r, k, v, ww, wb, u, gate, gn_w, gn_b = _fused_case(B, T, H, N, seed=74)
    shift = _rng(75).normal(size=H * N)
    a = oracle_mod.wkv6_fwd_fused(r, k, v, ww, wb, u, gate, gn_w, gn_b, 1e-5, H=H)
    b = oracle_mod.wkv6_fwd_fused(r, k, v, ww + shift, wb - shift, u, gate, gn_w, gn_b, 1e-5, H=H)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)
    c = oracle_mod.wkv6_fwd_fused(r, k, v, ww + shift, wb, u, gate, gn_w, gn_b, 1e-5, H=H)
    assert np.max(np.abs(c - a)) > 1e-3
