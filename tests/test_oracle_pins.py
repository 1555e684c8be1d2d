"""Pins of the float64 oracle against facts that do not come from the oracle itself.

Each test fixes one part of the oracle by a closed form, a hand-worked example,
brute force on a tiny case, an identity of the mathematics, or a special case
that reduces to a simpler formula. The combination is chosen so that a dropped
term, a wrong sign, a wrong index or a transposed operand anywhere in
oracle/moe.py fails at least one test here.
"""
import itertools
import math

import numpy as np
import pytest

from oracle import moe as om

RS = 1.5      # "route_scale": 1.5 (DeepSeek V4.1 inference/config.json)
LIM = 10.0    # "swiglu_limit": 10.0 (same file)


# ---------------------------------------------------------------- scalar functions
def test_softplus_closed_forms():
    assert om.softplus(0.0) == pytest.approx(math.log(2.0), abs=1e-16)
    assert om.sqrtsoftplus(0.0) == pytest.approx(math.sqrt(math.log(2.0)), abs=1e-16)
    # log(1+e^z) - log(1+e^-z) = z for every z
    for z in [-30.0, -3.5, -1.0, 0.25, 2.0, 17.0, 600.0]:
        assert om.softplus(z) - om.softplus(-z) == pytest.approx(z, rel=1e-14, abs=1e-14)
    # softplus(ln(e^a - 1)) = a: scores with a closed form
    for a in [0.25, 1.0, 4.0, 9.0]:
        z = math.log(math.expm1(a))
        assert om.softplus(z) == pytest.approx(a, rel=1e-13)
        assert om.sqrtsoftplus(z) == pytest.approx(math.sqrt(a), rel=1e-13)
    # tails: softplus(-50) = e^-50 to first order, softplus(800) = 800 without overflow
    assert om.softplus(-50.0) == pytest.approx(math.exp(-50.0), rel=1e-15)
    assert om.softplus(800.0) == 800.0
    assert np.all(np.diff(om.sqrtsoftplus(np.linspace(-40, 40, 2001))) > 0)   # strictly monotone


def test_silu_closed_forms():
    assert om.silu(0.0) == 0.0
    assert om.silu(1.0) == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), rel=1e-15)
    assert om.silu(-1.0) == pytest.approx(-1.0 / (1.0 + math.e), rel=1e-15)
    # silu(g) - silu(-g) = g
    for g in [-7.0, -0.3, 0.5, 3.0, 12.0]:
        assert om.silu(g) - om.silu(-g) == pytest.approx(g, rel=1e-14)
    with np.errstate(over="raise", invalid="raise", divide="raise"):
        assert om.silu(-800.0) == pytest.approx(0.0, abs=1e-300)
        assert om.silu(800.0) == 800.0


def test_clamp_directions():
    s10 = 10.0 / (1.0 + math.exp(-10.0))
    # gate is clamped from above only
    assert om.clamped_swiglu(20.0, 1.0, LIM) == pytest.approx(s10, rel=1e-15)
    assert om.clamped_swiglu(-20.0, 1.0, LIM) == pytest.approx(-20.0 / (1.0 + math.exp(20.0)), rel=1e-14)
    # up is clamped on both sides
    assert om.clamped_swiglu(1.0, 15.0, LIM) == pytest.approx(10.0 * om.silu(1.0), rel=1e-15)
    assert om.clamped_swiglu(1.0, -15.0, LIM) == pytest.approx(-10.0 * om.silu(1.0), rel=1e-15)
    # L = inf disables both clamps
    assert om.clamped_swiglu(20.0, -15.0, np.inf) == pytest.approx(-15.0 * om.silu(20.0), rel=1e-15)
    # L = 0: everything vanishes
    assert om.clamped_swiglu(3.0, 4.0, 0.0) == 0.0


# ---------------------------------------------------------------- routing
def _brute_topk(s, k):
    """Best k-subset by total score, ties by lexicographically smallest index tuple."""
    E = len(s)
    best, best_set = -np.inf, None
    for comb in itertools.combinations(range(E), k):
        v = sum(s[i] for i in comb)
        if v > best + 1e-15:
            best, best_set = v, comb
    return set(best_set)


@pytest.mark.parametrize("seed", range(6))
def test_topk_brute_force(seed):
    rng = np.random.default_rng(seed)
    E, H, T = 9, 5, 12
    x = rng.standard_normal((T, H))
    wg = rng.standard_normal((E, H)) / math.sqrt(H)
    for k in (1, 2, 4, 6):
        r = om.route(x, wg, k, RS)
        for t in range(T):
            assert set(r.idx[t]) == _brute_topk(r.s[t], k)
            sel = r.s[t, r.idx[t]]
            assert np.all(np.diff(sel) <= 0)                        # descending order
            assert r.w[t].sum() == pytest.approx(RS, rel=1e-14)     # weights sum to route_scale
            assert np.allclose(r.w[t], RS * sel / sel.sum(), rtol=1e-15)
            rest = np.delete(r.s[t], r.idx[t])
            assert r.gap[t] == pytest.approx(sel[-1] - rest.max(), abs=1e-15)


def test_topk_tie_breaks_to_lower_index():
    x = np.array([[1.0, 0.0]])
    wg = np.array([[0.5, 1.0], [2.0, 0.0], [0.5, -3.0], [2.0, 9.0], [-1.0, 0.0]])
    r = om.route(x, wg, 3, RS)
    # logits (0.5, 2, 0.5, 2, -1): two exact ties
    assert list(r.idx[0]) == [1, 3, 0]
    assert r.gap[0] == 0.0


def test_topk_order_matches_logit_order():
    # s is monotone in z, so top-k by s equals top-k by z
    rng = np.random.default_rng(7)
    x = rng.standard_normal((50, 16))
    wg = rng.standard_normal((40, 16)) / 4
    r = om.route(x, wg, 6, RS)
    assert np.array_equal(r.idx, np.argsort(-r.z, axis=1, kind="stable")[:, :6])


def test_bias_enters_the_logits():
    x = np.array([[1.0, 0.0]])
    wg = np.array([[1.0, 0.0], [0.9, 0.0], [0.0, 0.0]])
    b = np.array([0.0, 0.2, 0.0])
    r = om.route(x, wg, 1, RS, bias=b)
    assert list(r.idx[0]) == [1]
    assert r.z[0, 1] == pytest.approx(1.1)


# ---------------------------------------------------------------- hand-worked layer
def _hand_layer():
    """One token, H=4, E=4 routed + 1 shared, k=2, I=2, route_scale 1.5, L=10.

    x = e_0, so every projection reads column 0 of its [out, in] matrix; all the
    other entries are random and must not matter. The router column is chosen as
    z_e = ln(e^{a_e} - 1) so that s_e = sqrt(a_e) = (1, 3, 2, 0.5) exactly.
    """
    rng = np.random.default_rng(123)
    H, E, I = 4, 4, 2
    x = np.array([[1.0, 0.0, 0.0, 0.0]])
    wg = rng.standard_normal((E, H))
    wg[:, 0] = [math.log(math.expm1(a)) for a in (1.0, 9.0, 4.0, 0.25)]
    w1 = rng.standard_normal((E, I, H))
    w3 = rng.standard_normal((E, I, H))
    w2 = rng.standard_normal((E, H, I))
    w1[1][:, 0] = [2.0, -3.0];   w3[1][:, 0] = [1.0, 12.0]
    w2[1] = [[1, 0], [0, 1], [2, -1], [0, 0]]
    w1[2][:, 0] = [15.0, 0.0];   w3[2][:, 0] = [-0.5, 4.0]
    w2[2] = [[0, 1], [1, 0], [0, 0], [3, 0]]
    sh1 = rng.standard_normal((1, I, H)); sh3 = rng.standard_normal((1, I, H))
    sh2 = np.array([[[1, 1], [0, 0], [0, 0], [0, 2]]], dtype=np.float64)
    sh1[0][:, 0] = [1.0, -12.0]; sh3[0][:, 0] = [-12.0, 0.25]
    return x, wg, om.ExpertSource.from_arrays(w1, w3, w2, sh1, sh3, sh2)


def _silu(a):
    return a / (1.0 + math.exp(-a))


def test_hand_worked_layer():
    x, wg, ex = _hand_layer()
    res = om.moe_forward(x, wg, ex, k=2, route_scale=RS, limit=LIM)
    r = res.route
    assert np.allclose(r.s[0], [1.0, 3.0, 2.0, 0.5], rtol=1e-13)
    assert list(r.idx[0]) == [1, 2]
    assert np.allclose(r.w[0], [0.9, 0.6], rtol=1e-13)        # 1.5 * 3/5, 1.5 * 2/5
    # expert 1: G = (2, -3), U = (1, 12 -> 10)
    h1 = (_silu(2.0) * 1.0, _silu(-3.0) * 10.0)
    o1 = (h1[0], h1[1], 2 * h1[0] - h1[1], 0.0)
    # expert 2: G = (15 -> 10, 0), U = (-0.5, 4)
    h2 = (_silu(10.0) * -0.5, 0.0)
    o2 = (h2[1], h2[0], 0.0, 3 * h2[0])
    # shared: G = (1, -12) (no lower clamp on the gate), U = (-12 -> -10, 0.25)
    hs = (_silu(1.0) * -10.0, _silu(-12.0) * 0.25)
    osh = (hs[0] + hs[1], 0.0, 0.0, 2 * hs[1])
    expect = np.array(osh) + 0.9 * np.array(o1) + 0.6 * np.array(o2)
    assert np.allclose(res.y[0], expect, rtol=1e-13, atol=1e-15)


def test_expert_forward_loops():
    """Brute-force loops over the stored [out, in] layout on a tiny non-square expert."""
    rng = np.random.default_rng(3)
    n, H, I = 3, 7, 5
    x = rng.standard_normal((n, H))
    w1 = rng.standard_normal((I, H)); w3 = rng.standard_normal((I, H)) * 4
    w2 = rng.standard_normal((H, I))
    o, h = om.expert_forward(x, w1, w3, w2, 2.0)
    for t in range(n):
        hh = []
        for i in range(I):
            g = sum(x[t][c] * w1[i][c] for c in range(H))
            u = sum(x[t][c] * w3[i][c] for c in range(H))
            g = min(g, 2.0)
            u = max(-2.0, min(2.0, u))
            hh.append(_silu(g) * u)
        for c in range(H):
            assert o[t, c] == pytest.approx(sum(w2[c][i] * hh[i] for i in range(I)), rel=1e-12, abs=1e-13)
        assert np.allclose(h[t], hh, rtol=1e-13)


# ---------------------------------------------------------------- whole-layer invariants
def _rand_layer(seed, T=9, H=16, I=8, E=7, S=1):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H))
    wg = rng.standard_normal((E, H)) / math.sqrt(H)
    w1 = rng.standard_normal((E, I, H)) / math.sqrt(H) * 3
    w3 = rng.standard_normal((E, I, H)) / math.sqrt(H) * 3
    w2 = rng.standard_normal((E, H, I)) / math.sqrt(I)
    s1 = rng.standard_normal((S, I, H)) / math.sqrt(H) * 3
    s3 = rng.standard_normal((S, I, H)) / math.sqrt(H) * 3
    s2 = rng.standard_normal((S, H, I)) / math.sqrt(I)
    return x, wg, om.ExpertSource.from_arrays(w1, w3, w2, s1, s3, s2)


@pytest.mark.parametrize("seed", range(3))
def test_k_equals_E_reduces_to_dense_sum(seed):
    x, wg, ex = _rand_layer(seed)
    y = om.moe_forward(x, wg, ex, k=ex.n_routed, route_scale=RS, limit=np.inf).y
    yd = om.dense_reference(x, wg, ex, RS)
    assert np.allclose(y, yd, rtol=1e-12, atol=1e-13)
    # and the clamp does act on these inputs: with L = 1 the result differs
    y1 = om.moe_forward(x, wg, ex, k=ex.n_routed, route_scale=RS, limit=1.0).y
    assert not np.allclose(y1, yd, rtol=1e-6)


def test_token_permutation_invariance():
    x, wg, ex = _rand_layer(11, T=13)
    p = np.random.default_rng(0).permutation(13)
    y = om.moe_forward(x, wg, ex, 3, RS, LIM).y
    yp = om.moe_forward(x[p], wg, ex, 3, RS, LIM).y
    assert np.allclose(yp, y[p], rtol=1e-14, atol=1e-15)


def test_single_expert_special_case():
    # E = k = 1: weight = route_scale exactly, y = shared + 1.5 * expert_0
    x, wg, ex = _rand_layer(5, E=1)
    y = om.moe_forward(x, wg, ex, 1, RS, LIM).y
    o_sh = om.expert_forward(x, *ex.shared(0), LIM)[0]
    o_0 = om.expert_forward(x, *ex.routed(0), LIM)[0]
    assert np.allclose(y, o_sh + 1.5 * o_0, rtol=1e-14, atol=1e-15)


def test_zero_limit_gives_zero_output():
    x, wg, ex = _rand_layer(6)
    assert np.all(om.moe_forward(x, wg, ex, 3, RS, 0.0).y == 0.0)


def test_shared_expert_always_on_with_weight_one():
    # zero every routed W2: the output is the shared expert alone
    rng = np.random.default_rng(9)
    T, H, I, E = 5, 8, 4, 6
    x = rng.standard_normal((T, H)); wg = rng.standard_normal((E, H))
    w1 = rng.standard_normal((E, I, H)); w3 = rng.standard_normal((E, I, H))
    w2 = np.zeros((E, H, I))
    s1 = rng.standard_normal((1, I, H)); s3 = rng.standard_normal((1, I, H)); s2 = rng.standard_normal((1, H, I))
    ex = om.ExpertSource.from_arrays(w1, w3, w2, s1, s3, s2)
    y = om.moe_forward(x, wg, ex, 2, RS, LIM).y
    assert np.allclose(y, om.expert_forward(x, s1[0], s3[0], s2[0], LIM)[0], rtol=1e-15)


def _layer_with_shared(S, seed=11):
    rng = np.random.default_rng(seed)
    T, H, I, E = 5, 8, 4, 6
    x = rng.standard_normal((T, H)); wg = rng.standard_normal((E, H))
    w1 = rng.standard_normal((E, I, H)); w3 = rng.standard_normal((E, I, H)); w2 = rng.standard_normal((E, H, I))
    s1 = rng.standard_normal((S, I, H)); s3 = rng.standard_normal((S, I, H)); s2 = rng.standard_normal((S, H, I))
    return x, wg, (w1, w3, w2), (s1, s3, s2)


def test_no_shared_expert_is_the_routed_sum():
    # n_shared = 0: y is the weighted sum over the selected experts, written out here
    x, wg, (w1, w3, w2), (s1, s3, s2) = _layer_with_shared(0)
    ex = om.ExpertSource.from_arrays(w1, w3, w2, s1, s3, s2)
    res = om.moe_forward(x, wg, ex, 2, RS, LIM)
    want = np.zeros_like(x)
    for t in range(x.shape[0]):
        for j in range(2):
            e = res.route.idx[t, j]
            want[t] += res.route.w[t, j] * om.expert_forward(x[t:t + 1], w1[e], w3[e], w2[e], LIM)[0][0]
    assert np.allclose(res.y, want, rtol=1e-13, atol=1e-13)


def test_each_shared_expert_adds_with_weight_one():
    # two shared experts: one with W2 = 0 changes nothing; a copy of the first
    # adds the same contribution again
    x, wg, routed, (s1, s3, s2) = _layer_with_shared(1)
    one = om.moe_forward(x, wg, om.ExpertSource.from_arrays(*routed, s1, s3, s2), 2, RS, LIM).y
    zero2 = (np.concatenate([s1, s1]), np.concatenate([s3, s3]), np.concatenate([s2, np.zeros_like(s2)]))
    with_zero = om.moe_forward(x, wg, om.ExpertSource.from_arrays(*routed, *zero2), 2, RS, LIM).y
    assert np.allclose(with_zero, one, rtol=1e-15, atol=1e-15)
    twice = (np.concatenate([s1, s1]), np.concatenate([s3, s3]), np.concatenate([s2, s2]))
    doubled = om.moe_forward(x, wg, om.ExpertSource.from_arrays(*routed, *twice), 2, RS, LIM).y
    shared = om.expert_forward(x, s1[0], s3[0], s2[0], LIM)[0]
    assert np.allclose(doubled - one, shared, rtol=1e-12, atol=1e-12)


def test_permutation_reference_brute_force():
    rng = np.random.default_rng(2)
    T, k, E = 11, 3, 5
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)])
    counts, offsets, perm, inv = om.permutation_reference(idx, E)
    expected = [t * k + j for e in range(E) for t in range(T) for j in range(k) if idx[t, j] == e]
    assert list(perm) == expected
    assert counts.sum() == T * k and offsets[-1] == T * k
    for e in range(E):
        assert np.all(idx.reshape(-1)[perm[offsets[e]:offsets[e + 1]]] == e)
    assert np.array_equal(perm[inv], np.arange(T * k))
