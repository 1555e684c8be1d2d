"""Pins of the oracle's expert-parallel decomposition (MAX DeepseekV41Config
ep_config; the DEP recipes on the DeepSeek-V4-Pro page): every rank routes all
tokens with the full router and sums only the slots whose expert lies in its
window of the experts (plus the shared experts on exactly one rank)."""
import numpy as np
import pytest

from oracle import moe as om

from test_oracle_pins import LIM, RS, _hand_layer


def _layer(seed, T=7, H=16, I=8, E=12, S=1):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H))
    wg = rng.standard_normal((E, H)) / 4
    ex = om.ExpertSource.from_arrays(rng.standard_normal((E, I, H)) / 4, rng.standard_normal((E, I, H)) / 4,
                                     rng.standard_normal((E, H, I)) / 3, rng.standard_normal((S, I, H)) / 4,
                                     rng.standard_normal((S, I, H)) / 4, rng.standard_normal((S, H, I)) / 3)
    return x, wg, ex


@pytest.mark.parametrize("cuts", [[0, 12], [0, 6, 12], [0, 3, 4, 9, 12], [0, 0, 12], [0, 12, 12]])
def test_windows_of_a_partition_sum_to_the_layer(cuts):
    x, wg, ex = _layer(1)
    full = om.moe_forward(x, wg, ex, 3, RS, LIM).y
    parts = [om.moe_forward_partial(x, wg, ex, 3, RS, LIM, a, b, include_shared=(i == 0))
             for i, (a, b) in enumerate(zip(cuts[:-1], cuts[1:]))]
    assert np.allclose(sum(parts), full, rtol=1e-12, atol=1e-14)


def test_hand_worked_windows():
    """The hand-worked layer selects experts 1 and 2 at weights 0.9 and 0.6: the
    window [0, 2) holds 0.9 expert_1 alone, [2, 4) holds 0.6 expert_2 alone."""
    x, wg, ex = _hand_layer()
    o1 = om.expert_forward(x, *ex.routed(1), LIM)[0]
    o2 = om.expert_forward(x, *ex.routed(2), LIM)[0]
    osh = om.expert_forward(x, *ex.shared(0), LIM)[0]
    lo = om.moe_forward_partial(x, wg, ex, 2, RS, LIM, 0, 2, include_shared=False)
    hi = om.moe_forward_partial(x, wg, ex, 2, RS, LIM, 2, 4, include_shared=True)
    assert np.allclose(lo, 0.9 * o1, rtol=1e-14)
    assert np.allclose(hi, osh + 0.6 * o2, rtol=1e-14)
    # a window no token selects contributes nothing
    assert not np.any(om.moe_forward_partial(x, wg, ex, 2, RS, LIM, 3, 4, include_shared=False))
