"""Pins of the oracle's MX mirror dispatch: with MXFP4 routed experts, which parts
of the layer see MXFP8-quantised activations.

The reading pinned here (MXFP4 routed experts, "expert_dtype": "fp4" of the
DeepSeek V4.1 inference/config.json; shared expert and router in BF16): the
router and the shared expert see the token as given; a routed expert sees the
token quantised to MXFP8 (E4M3, E8M0 per 32 along the hidden dimension) and its
own SwiGLU output quantised the same way along the expert width.

Each test builds inputs whose outcome under that reading follows from the
MXFP8 block rule alone (pinned separately in test_oracle_mx.py): two tokens
that differ only below the E4M3 resolution of their block must give bit-equal
routed outputs, a router near-tie that quantisation would flip must not flip,
and a layer whose routed experts output zero must equal the BF16 layer. Each
test also checks that its construction would expose the opposite reading, so a
plausible mistake (quantising the shared expert or the router input, or not
quantising a routed expert's x or h) fails at least one of them.
"""
import numpy as np

from oracle import moe as om
from oracle import mx

H, I = 64, 32          # two MX blocks along H, one along I


def _source(w1, w3, w2, sh_w1, sh_w3, sh_w2, routed_is_mx=True):
    """Expert source that declares its routed experts MXFP4 (the dispatch under test)."""
    src = om.ExpertSource.from_arrays(w1, w3, w2, sh_w1, sh_w3, sh_w2)
    src.routed_is_mx = routed_is_mx
    return src


def _layer(rng, E=4, S=1):
    w1 = rng.standard_normal((E, I, H)) / 8
    w3 = rng.standard_normal((E, I, H)) / 8
    w2 = rng.standard_normal((E, H, I)) / 6
    sh = (rng.standard_normal((S, I, H)) / 8, rng.standard_normal((S, I, H)) / 8,
          rng.standard_normal((S, H, I)) / 6)
    return w1, w3, w2, sh


def test_router_sees_the_unquantised_token():
    # Coordinate 0 holds 1 + 2^-5, which MXFP8 rounds to 1.0 in a block whose
    # amax is 1.75 (scale 2^-8, E4M3 step 32 at 264). Expert 0's logit is x0,
    # expert 1's is 1.015625 * x2 with x2 = 1 on the grid: unquantised, expert
    # 0 wins (1.03125 > 1.015625); quantised, expert 1 would.
    x = np.zeros((1, H))
    x[0, 0], x[0, 1], x[0, 2] = 1.0 + 2.0 ** -5, 1.75, 1.0
    assert mx.mx_roundtrip(x, "e4m3")[0, 0] == 1.0
    wg = np.zeros((4, H))
    wg[0, 0] = 1.0
    wg[1, 2] = 1.015625
    rng = np.random.default_rng(1)
    w1, w3, w2, sh = _layer(rng)
    res = om.moe_forward(x, wg, _source(w1, w3, w2, *sh), 1, 1.5, 10.0)
    assert res.route.idx[0, 0] == 0
    # the construction is sensitive: routing the quantised token picks expert 1
    assert om.route(mx.mx_roundtrip(x, "e4m3"), wg, 1, 1.5).idx[0, 0] == 1
    # and the MXFP4 layer's routing is the BF16 layer's, bit for bit
    ref = om.moe_forward(x, wg, _source(w1, w3, w2, *sh, routed_is_mx=False), 1, 1.5, 10.0)
    assert np.array_equal(res.route.z, ref.route.z) and np.array_equal(res.route.w, ref.route.w)


def test_shared_expert_sees_the_unquantised_token():
    # Routed experts whose down projection is zero contribute exactly 0, so the
    # MXFP4 layer's output must be the BF16 layer's output bit for bit: the
    # shared expert alone, on the token as given.
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, H))                     # off the MXFP8 grid
    assert not np.array_equal(mx.mx_roundtrip(x, "e4m3"), x)
    wg = rng.standard_normal((4, H)) / 8
    w1, w3, w2, sh = _layer(rng)
    w2 = np.zeros_like(w2)
    y_mx = om.moe_forward(x, wg, _source(w1, w3, w2, *sh), 2, 1.5, 10.0).y
    y_bf = om.moe_forward(x, wg, _source(w1, w3, w2, *sh, routed_is_mx=False), 2, 1.5, 10.0).y
    assert np.array_equal(y_mx, y_bf)
    # sensitive: the shared expert on the quantised token differs
    o_q = om.expert_forward(mx.mx_roundtrip(x, "e4m3"), sh[0][0], sh[1][0], sh[2][0], 10.0)[0]
    assert not np.allclose(o_q, y_bf, rtol=1e-9, atol=0)


def test_routed_experts_see_the_quantised_token():
    # Tokens a and b differ only in coordinate 3 (1 + 2^-5 against 1.0) inside a
    # block with amax 1.75, where MXFP8 maps both to 1.0. The router ignores that
    # coordinate (equal logits, equal weights) and the shared expert's output is
    # zero, so a routed expert fed the quantised token gives bit-equal rows.
    rng = np.random.default_rng(3)
    base = mx.mx_roundtrip(rng.standard_normal(H), "e4m3")
    base[0:32] = np.where(np.abs(base[0:32]) > 1.75, np.sign(base[0:32]) * 1.5, base[0:32])
    base[5] = 1.75
    x = np.stack([base, base])
    x[0, 3], x[1, 3] = 1.0 + 2.0 ** -5, 1.0
    xq = mx.mx_roundtrip(x, "e4m3")
    assert np.array_equal(xq[0], xq[1]) and not np.array_equal(x[0], x[1])
    wg = rng.standard_normal((4, H)) / 8
    wg[:, 3] = 0.0
    w1, w3, w2, sh = _layer(rng)
    sh = (sh[0], sh[1], np.zeros_like(sh[2]))
    y = om.moe_forward(x, wg, _source(w1, w3, w2, *sh), 2, 1.5, 10.0).y
    assert np.array_equal(y[0], y[1])
    # sensitive: the same layer with BF16 routed experts tells the tokens apart
    y_bf = om.moe_forward(x, wg, _source(w1, w3, w2, *sh, routed_is_mx=False), 2, 1.5, 10.0).y
    assert not np.array_equal(y_bf[0], y_bf[1])


def test_routed_experts_see_the_quantised_swiglu_output():
    # Tokens on the MXFP8 grid (so x is not changed by quantisation) that differ
    # only in coordinate d, which reaches the expert only through h_1 = silu(1) *
    # 2^-20 * x_d (below 2e-6). h_0 = silu(10) * 8 is about 80, so the block of h
    # has scale 2^-2 and its smallest E4M3 step is 2^-11 (5e-4): both h_1 round
    # to 0 and the two tokens' routed outputs must be bit-equal.
    d, c, e_u, f = 40, 1, 2, 7
    x = np.zeros((2, H))
    for t in range(2):
        x[t, c] = x[t, e_u] = x[t, f] = 1.0
    x[0, d], x[1, d] = 1.0, 2.0
    assert np.array_equal(mx.mx_roundtrip(x, "e4m3"), x)
    E = 4
    wg = np.zeros((E, H))
    wg[:, f] = [0.5, 0.25, -0.25, 0.125]                # router ignores coordinate d
    w1 = np.zeros((E, I, H)); w3 = np.zeros((E, I, H)); w2 = np.zeros((E, H, I))
    w1[:, 0, c] = 10.0                                   # g_0 = 10 (clamped at L = 10)
    w3[:, 0, e_u] = 8.0                                  # u_0 = 8
    w1[:, 1, c] = 1.0                                    # g_1 = 1
    w3[:, 1, d] = 2.0 ** -20                             # u_1 = 2^-20 x_d
    w2[:, :, 1] = 1.0                                    # every output reads h_1 ...
    w2[:, 0, 0] = 1.0                                    # ... and output 0 also h_0
    S = 1
    sh = (np.zeros((S, I, H)), np.zeros((S, I, H)), np.zeros((S, H, I)))
    h = om.expert_forward(x, w1[0], w3[0], w2[0], 10.0)[1]
    assert 0 < h[0, 1] < h[1, 1] < 2e-6 and 79.99 < h[0, 0] < 80.0
    hq = mx.mx_roundtrip(h, "e4m3")
    assert np.array_equal(hq[0], hq[1]) and hq[0, 1] == 0.0
    y = om.moe_forward(x, wg, _source(w1, w3, w2, *sh), 2, 1.5, 10.0).y
    assert np.array_equal(y[0], y[1])
    assert y[0, 0] != 0.0                                # the routed path is live
    y_bf = om.moe_forward(x, wg, _source(w1, w3, w2, *sh, routed_is_mx=False), 2, 1.5, 10.0).y
    assert not np.array_equal(y_bf[0], y_bf[1])


def test_mxfp4_expert_source_serves_the_stored_values():
    # from_mxfp4 hands out the exact values the packed bytes encode (the MXFP4
    # round trip of the weights it was packed from), marks the routed experts
    # MXFP4, and serves the shared expert unchanged.
    rng = np.random.default_rng(5)
    E, S = 3, 1
    w = [rng.standard_normal((E, I, H)) / 8, rng.standard_normal((E, I, H)) / 8, rng.standard_normal((E, H, I)) / 6]
    packed = [mx.quantize_mxfp4_packed(a) for a in w]
    sh = [rng.standard_normal((S, I, H)), rng.standard_normal((S, I, H)), rng.standard_normal((S, H, I))]
    src = om.ExpertSource.from_mxfp4(packed[0][0], packed[0][1], packed[1][0], packed[1][1],
                                     packed[2][0], packed[2][1], *sh)
    assert src.routed_is_mx and src.n_routed == E and src.n_shared == S
    for e in range(E):
        for got, ref in zip(src.routed(e), w):
            assert np.array_equal(got, mx.mx_roundtrip(ref[e], "e2m1"))
    for got, ref in zip(src.shared(0), sh):
        assert np.array_equal(got, ref[0])
