"""Pins of the oracle's hash routing (MAX DeepseekV41Config num_hash_layers; the
DeepSeek-V4-Pro config paragraph's "num_hash_layers 3").

Reading pinned: a hash layer's k experts are the row of a fixed vocabulary table
selected by the token's id, in the table's order; their weights are the
sqrtsoftplus scores of those experts normalised over the k and scaled by
route_scale. The hand-worked layer of test_oracle_pins.py (scores 1, 3, 2, 0.5
exactly) gives closed-form weights and outputs for any table row.
"""
import numpy as np

from oracle import moe as om

from test_oracle_pins import LIM, RS, _hand_layer, _silu


def _hand_expect():
    """The hand-worked layer's output with experts 1 and 2 at weights 0.9 and 0.6,
    and the two experts' outputs alone (written out in test_hand_worked_layer)."""
    h1 = (_silu(2.0) * 1.0, _silu(-3.0) * 10.0)
    o1 = np.array((h1[0], h1[1], 2 * h1[0] - h1[1], 0.0))
    h2 = (_silu(10.0) * -0.5, 0.0)
    o2 = np.array((h2[1], h2[0], 0.0, 3 * h2[0]))
    hs = (_silu(1.0) * -10.0, _silu(-12.0) * 0.25)
    osh = np.array((hs[0] + hs[1], 0.0, 0.0, 2 * hs[1]))
    return osh, o1, o2


def test_table_row_selects_and_scores_weight():
    x, wg, ex = _hand_layer()
    table = np.array([[0, 1], [2, 1], [3, 0]])
    # token id 1 -> experts (2, 1): weights 1.5 * (2, 3) / 5
    res = om.moe_forward_hashed(x, wg, ex, table, [1], RS, LIM)
    assert list(res.route.idx[0]) == [2, 1]
    assert np.allclose(res.route.w[0], [0.6, 0.9], rtol=1e-13)
    osh, o1, o2 = _hand_expect()
    assert np.allclose(res.y[0], osh + 0.9 * o1 + 0.6 * o2, rtol=1e-13, atol=1e-15)
    # token id 2 -> experts (3, 0), which the learned router would never pick: 1.5 * (0.5, 1) / 1.5
    r = om.hash_route(x, wg, table, [2], RS)
    assert list(r.idx[0]) == [3, 0]
    assert np.allclose(r.w[0], [0.5, 1.0], rtol=1e-13)
    assert np.isclose(r.w.sum(), RS, rtol=1e-14)


def test_selection_does_not_depend_on_the_router():
    rng = np.random.default_rng(3)
    T, H, E, k = 6, 16, 10, 3
    x = rng.standard_normal((T, H))
    table = np.array([rng.permutation(E)[:k] for _ in range(20)])
    ids = rng.integers(0, 20, size=T)
    r1 = om.hash_route(x, rng.standard_normal((E, H)), table, ids, RS)
    r2 = om.hash_route(x, rng.standard_normal((E, H)), table, ids, RS)
    assert np.array_equal(r1.idx, table[ids]) and np.array_equal(r2.idx, table[ids])
    assert not np.allclose(r1.w, r2.w)
    assert np.allclose(r1.w.sum(axis=1), RS, rtol=1e-14)


def test_table_of_the_learned_choice_gives_the_learned_layer():
    rng = np.random.default_rng(4)
    T, H, I, E, k = 5, 16, 8, 6, 2
    x = rng.standard_normal((T, H))
    wg = rng.standard_normal((E, H)) / 4
    ex = om.ExpertSource.from_arrays(rng.standard_normal((E, I, H)) / 4, rng.standard_normal((E, I, H)) / 4,
                                     rng.standard_normal((E, H, I)) / 3, rng.standard_normal((1, I, H)) / 4,
                                     rng.standard_normal((1, I, H)) / 4, rng.standard_normal((1, H, I)) / 3)
    learned = om.moe_forward(x, wg, ex, k, RS, LIM)
    table = learned.route.idx                 # token id t -> the learned top-k of token t
    hashed = om.moe_forward_hashed(x, wg, ex, table, np.arange(T), RS, LIM)
    assert np.array_equal(hashed.y, learned.y) and np.array_equal(hashed.route.w, learned.route.w)
    # ids, not token positions, pick the row: permuting tokens with their ids permutes y
    p = rng.permutation(T)
    hp = om.moe_forward_hashed(x[p], wg, ex, table, p, RS, LIM)
    assert np.allclose(hp.y, learned.y[p], rtol=1e-13, atol=1e-15)
    # the same token under another id gets that id's experts
    other = om.hash_route(x[:1], wg, table, [T - 1], RS)
    assert np.array_equal(other.idx[0], table[T - 1])
