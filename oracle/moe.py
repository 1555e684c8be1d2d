"""Plain float64 CPU oracle of the DeepSeek-V4.1-Flash routed-expert FFN layer.

TEST INFRASTRUCTURE ONLY. It is slow on purpose and shares no code with the
CUDA path; the product never imports it. Only tests/, __graft_entry__.smoke()
and bench.py (its cpu_baseline leg and its ``--impl reference`` arm) use it.

What the pages fix:
  * routed experts 384, shared experts 1, 6 active per token, hidden 5120,
    expert width 2304 (DeepSeek V4.1 inference/config.json: "n_routed_experts",
    "n_shared_experts", "n_activated_experts", "dim", "moe_inter_dim"; MAX
    DeepseekV41Config fields n_routed_experts, num_experts_per_tok,
    moe_intermediate_size);
  * "score_func": "sqrtsoftplus", "route_scale": 1.5, "swiglu_limit": 10.0
    (inference/config.json; MAX routed_scaling_factor / swiglu_limit);
  * experts are gated MLPs and the shared expert has the routed experts' width
    (llm-architectures-explained "DeepSeek-V4.1-Flash", "Every architecture
    field" table: ffns.moe.gated, ffns.moe.d_shared).

The pages name the scoring function and the clamp but print no formula. The
formulas below are the plainest reading, fixed as follows:
    z_e   = x . Wg_e (+ b_e)
    s_e   = sqrt(softplus(z_e)),  softplus(z) = log(1 + e^z)
    top-k = the k largest s_e (ties: lower expert index first), in descending order
    w_j   = route_scale * s_(j) / sum_{selected} s
    expert(x) = W2 (silu(min(W1 x, L)) * clamp(W3 x, -L, L))
    y     = sum_shared expert_sh(x) + sum_j w_j expert_(j)(x)
Matrices are stored [out, in] (row-major, input dimension contiguous), so
W1 x is ``w1 @ x`` for one token and ``x @ w1.T`` for a batch of rows.

MX mirror mode (routed experts in MXFP4 or MXFP8): the routed experts see the token
quantised to MXFP8 (E4M3, one E8M0 scale per 32 along the hidden dimension)
and the SwiGLU output h quantised the same way along the expert width; the
router and the shared expert see the unquantised BF16 values.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Callable, Optional, Sequence

import numpy as np

from . import mx


# ----------------------------------------------------------------------------
# scalar functions
# ----------------------------------------------------------------------------
def softplus(z):
    """log(1 + e^z), in the overflow-free form max(z, 0) + log1p(e^-|z|)."""
    z = np.asarray(z, dtype=np.float64)
    return np.maximum(z, 0.0) + np.log1p(np.exp(-np.abs(z)))


def sqrtsoftplus(z):
    """The "sqrtsoftplus" routing score: sqrt(softplus(z))."""
    return np.sqrt(softplus(z))


def silu(g):
    """g * sigmoid(g) = g / (1 + e^-g), evaluated without overflow for g << 0."""
    g = np.asarray(g, dtype=np.float64)
    # For g < 0 write sigmoid(g) = e^g / (1 + e^g) so e^-g never overflows.
    eg = np.exp(-np.abs(g))
    sig = np.where(g >= 0, 1.0 / (1.0 + eg), eg / (1.0 + eg))
    return g * sig


def clamped_swiglu(g, u, limit):
    """silu(min(g, L)) * clamp(u, -L, L); limit = inf disables both clamps."""
    g = np.asarray(g, dtype=np.float64)
    u = np.asarray(u, dtype=np.float64)
    if np.isfinite(limit):
        g = np.minimum(g, limit)
        u = np.clip(u, -limit, limit)
    return silu(g) * u


# ----------------------------------------------------------------------------
# routing
# ----------------------------------------------------------------------------
@dataclass
class Route:
    z: np.ndarray        # [T, E] logits (bias included)
    s: np.ndarray        # [T, E] scores
    idx: np.ndarray      # [T, k] int64, descending score
    w: np.ndarray        # [T, k] weights, sum = route_scale per token
    gap: np.ndarray      # [T] s_(k) - s_(k+1) (inf when k == E)


def route(x, wg, k, route_scale, bias=None, idx_override=None):
    """Router logits, sqrtsoftplus scores, top-k and normalised weights.

    x [T, H], wg [E, H], bias [E] or None. If idx_override [T, k] is given the
    selection is taken from it (used to re-evaluate near-tie tokens with the
    indices another implementation picked) and the weights follow from it.
    """
    x = np.asarray(x, dtype=np.float64)
    wg = np.asarray(wg, dtype=np.float64)
    z = x @ wg.T
    if bias is not None:
        z = z + np.asarray(bias, dtype=np.float64)[None, :]
    s = sqrtsoftplus(z)
    T, E = s.shape
    if not (1 <= k <= E):
        raise ValueError("need 1 <= k <= E")
    # Stable ordering: descending score, ties broken by ascending expert index.
    order = np.lexsort((np.broadcast_to(np.arange(E), (T, E)), -s), axis=-1)
    sorted_s = np.take_along_axis(s, order, axis=-1)
    gap = sorted_s[:, k - 1] - sorted_s[:, k] if k < E else np.full(T, np.inf)
    idx = order[:, :k] if idx_override is None else np.asarray(idx_override, dtype=np.int64)
    s_sel = np.take_along_axis(s, idx, axis=-1)
    w = route_scale * s_sel / s_sel.sum(axis=-1, keepdims=True)
    return Route(z=z, s=s, idx=idx, w=w, gap=gap)


def hash_route(x, wg, table, token_ids, route_scale, bias=None):
    """Routing of a hash layer (MAX DeepseekV41Config num_hash_layers; the
    DeepSeek-V4-Pro config paragraph: "num_hash_layers 3").

    The pages name hash layers but give no hash function. Reading adopted: a hash
    layer takes its k experts from a fixed table of the vocabulary,
    table [vocab, k] of distinct expert indices (a layer weight, like the router),
    row token_ids[t] for token t, in the table's order, in place of the router's
    top-k; the weights are the sqrtsoftplus scores of those experts, normalised
    over the k and scaled by route_scale, exactly as for learned routing.
    """
    table = np.asarray(table, dtype=np.int64)
    token_ids = np.asarray(token_ids, dtype=np.int64)
    sel = table[token_ids]
    return route(x, wg, sel.shape[1], route_scale, bias=bias, idx_override=sel)


def moe_forward_hashed(x, wg, experts, table, token_ids, route_scale, limit, bias=None, mx_act=None):
    """The layer with hash routing: the selection of hash_route, everything else as moe_forward."""
    table = np.asarray(table, dtype=np.int64)
    sel = table[np.asarray(token_ids, dtype=np.int64)]
    return moe_forward(x, wg, experts, sel.shape[1], route_scale, limit, bias=bias, idx_override=sel,
                       mx_act=mx_act)


# ----------------------------------------------------------------------------
# experts
# ----------------------------------------------------------------------------
def expert_forward(x, w1, w3, w2, limit, mx_act=False):
    """One gated expert on rows x [n, H]: returns (o [n, H], h [n, I]).

    With mx_act the input rows and h are replaced by their MXFP8 round trip
    (the values an MXFP8 x MXFP4 tensor-core path consumes).
    """
    x = np.asarray(x, dtype=np.float64)
    if mx_act:
        x = mx.mx_roundtrip(x, "e4m3")
    g = x @ np.asarray(w1, dtype=np.float64).T
    u = x @ np.asarray(w3, dtype=np.float64).T
    h = clamped_swiglu(g, u, limit)
    hh = mx.mx_roundtrip(h, "e4m3") if mx_act else h
    o = hh @ np.asarray(w2, dtype=np.float64).T
    return o, h


class ExpertSource:
    """Gives float64 expert matrices on demand (so a 27 GB layer need not be resident).

    routed(e) -> (w1 [I,H], w3 [I,H], w2 [H,I]); shared(j) -> same for shared expert j.
    """

    def __init__(self, routed: Callable[[int], tuple], shared: Callable[[int], tuple],
                 n_routed: int, n_shared: int, routed_is_mx: bool = False):
        self.routed = routed
        self.shared = shared
        self.n_routed = n_routed
        self.n_shared = n_shared
        self.routed_is_mx = routed_is_mx

    @staticmethod
    def from_arrays(w1, w3, w2, sh_w1, sh_w3, sh_w2):
        """BF16/float arrays [E, I, H], [E, I, H], [E, H, I] (+ shared [S, ...])."""
        f = lambda a, e: np.asarray(a[e], dtype=np.float64)
        return ExpertSource(lambda e: (f(w1, e), f(w3, e), f(w2, e)),
                            lambda j: (f(sh_w1, j), f(sh_w3, j), f(sh_w2, j)),
                            len(w1), len(sh_w1))

    @staticmethod
    def from_mxfp4(q1, s1, q3, s3, q2, s2, sh_w1, sh_w3, sh_w2):
        """Packed E2M1 [E, I, H/2] / E8M0 [E, I, H/32] (etc.) routed, BF16 shared."""
        dq = mx.dequantize_mxfp4_packed
        f = lambda a, e: np.asarray(a[e], dtype=np.float64)
        return ExpertSource(
            lambda e: (dq(q1[e], s1[e]), dq(q3[e], s3[e]), dq(q2[e], s2[e])),
            lambda j: (f(sh_w1, j), f(sh_w3, j), f(sh_w2, j)),
            len(q1), len(sh_w1), routed_is_mx=True)


    @staticmethod
    def from_mxfp8(q1, s1, q3, s3, q2, s2, sh_w1, sh_w3, sh_w2):
        """E4M3 codes [E, I, H] / E8M0 [E, I, H/32] (etc.) routed, BF16 shared.

        Routed experts stored in a block-scaled 8-bit format meet MXFP8 activations
        like the MXFP4 ones, so they are marked for the MX mirror as well."""
        dq = mx.dequantize_mxfp8
        f = lambda a, e: np.asarray(a[e], dtype=np.float64)
        return ExpertSource(
            lambda e: (dq(q1[e], s1[e]), dq(q3[e], s3[e]), dq(q2[e], s2[e])),
            lambda j: (f(sh_w1, j), f(sh_w3, j), f(sh_w2, j)),
            len(q1), len(sh_w1), routed_is_mx=True)


@dataclass
class MoEResult:
    y: np.ndarray            # [T, H]
    route: Route
    h_shared: list = field(default_factory=list)   # per shared expert: h [T, I]


def moe_forward(x, wg, experts: ExpertSource, k, route_scale, limit, bias=None,
                idx_override=None, mx_act: Optional[bool] = None, keep_h=False):
    """The whole layer on token rows x [T, H] (float64 accumulation throughout).

    mx_act defaults to experts.routed_is_mx: routed experts stored in MXFP4 see
    MXFP8-quantised activations; shared experts never do.
    """
    x = np.asarray(x, dtype=np.float64)
    if mx_act is None:
        mx_act = experts.routed_is_mx
    r = route(x, wg, k, route_scale, bias=bias, idx_override=idx_override)
    T, H = x.shape
    y = np.zeros((T, H), dtype=np.float64)
    res = MoEResult(y=y, route=r)
    for j in range(experts.n_shared):
        w1, w3, w2 = experts.shared(j)
        o, h = expert_forward(x, w1, w3, w2, limit, mx_act=False)
        y += o
        if keep_h:
            res.h_shared.append(h)
    # Routed experts: visit each expert once with all of its (token, slot) rows.
    for e in np.unique(r.idx):
        tok, slot = np.nonzero(r.idx == e)
        w1, w3, w2 = experts.routed(int(e))
        o, _ = expert_forward(x[tok], w1, w3, w2, limit, mx_act=mx_act)
        # A token selects an expert at most once, so the rows in tok are distinct.
        y[tok] += r.w[tok, slot][:, None] * o
    return res


def moe_forward_partial(x, wg, experts: ExpertSource, k, route_scale, limit, expert_begin, expert_end,
                        include_shared, bias=None, mx_act: Optional[bool] = None):
    """One rank's share of an expert-parallel layer (MAX DeepseekV41Config ep_config,
    "only under data parallelism"; the DEP recipes on the DeepSeek-V4-Pro page).

    The experts are split into windows [expert_begin, expert_end), one per rank;
    every rank routes all tokens with the full router. A rank's partial output is
    the weighted sum over the selected slots whose expert lies in its window, plus
    the shared experts when include_shared (exactly one rank holds them). The
    partial outputs of a partition of [0, E) sum to the layer's output.
    """
    x = np.asarray(x, dtype=np.float64)
    if mx_act is None:
        mx_act = experts.routed_is_mx
    r = route(x, wg, k, route_scale, bias=bias)
    y = np.zeros_like(x)
    if include_shared:
        for j in range(experts.n_shared):
            y += expert_forward(x, *experts.shared(j), limit, mx_act=False)[0]
    for e in np.unique(r.idx):
        if not (expert_begin <= e < expert_end):
            continue
        tok, slot = np.nonzero(r.idx == e)
        o, _ = expert_forward(x[tok], *experts.routed(int(e)), limit, mx_act=mx_act)
        y[tok] += r.w[tok, slot][:, None] * o
    return y


def dense_reference(x, wg, experts: ExpertSource, route_scale, bias=None):
    """The k = E, L = inf special case written without any top-k code:

        y = sum_sh expert_sh(x) + route_scale * sum_e (s_e / sum_all s) expert_e(x)

    Used to pin moe_forward: with every expert selected and the clamp disabled the
    two must agree to rounding.
    """
    x = np.asarray(x, dtype=np.float64)
    z = x @ np.asarray(wg, dtype=np.float64).T
    if bias is not None:
        z = z + np.asarray(bias, dtype=np.float64)[None, :]
    s = sqrtsoftplus(z)
    frac = s / s.sum(axis=-1, keepdims=True)
    y = np.zeros_like(x)
    for j in range(experts.n_shared):
        y += expert_forward(x, *experts.shared(j), np.inf)[0]
    for e in range(experts.n_routed):
        y += route_scale * frac[:, e:e + 1] * expert_forward(x, *experts.routed(e), np.inf)[0]
    return y


def permutation_reference(idx, n_routed):
    """Expert-major order of (token, slot) pairs, ascending (token, slot) inside an expert.

    Returns (counts [E], offsets [E+1], perm [T*k] of flat slot ids, inv [T*k]).
    """
    idx = np.asarray(idx, dtype=np.int64)
    flat = idx.reshape(-1)
    counts = np.bincount(flat, minlength=n_routed).astype(np.int64)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    perm = np.argsort(flat, kind="stable")      # stable: ties keep ascending flat id
    inv = np.empty_like(perm)
    inv[perm] = np.arange(len(perm))
    return counts, offsets, perm, inv
