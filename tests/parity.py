"""Parity helpers: run the oracle on the same seeded inputs and compare.

Tolerances (fixed before any kernel ran):
  * routing: for every token whose oracle gap s_(k) - s_(k+1) exceeds 1e-6 the
    selected experts must equal the oracle's, in the same descending order;
    tokens at or below that gap may pick differently, and their oracle output
    is recomputed with the GPU's choice;
  * routing weights: |w_gpu - w_oracle| <= 1e-5 (fp32 rounding of an fp64 value);
  * layer output, element by element: |y_gpu - y_oracle| <= 2e-2 * RMS(y_oracle)
    + 2^-8 |y_oracle| over the compared rows. The GPU rounds h and y to BF16 and
    accumulates in fp32; the second term covers the rounding of y itself (2^-9 of
    |y|, twice), which the largest elements (about 5 RMS) need: the float64 layer
    with only h and y rounded to BF16 reaches 2.0-2.7 % of RMS at such elements for
    some shapes (small expert widths, many compared elements);
  * BF16 SwiGLU rows h, element by element: |h_gpu - h_oracle| <= 2^-8 |h_oracle|
    + 1e-3 RMS(h_oracle) (h is stored in BF16, whose rounding is 2^-9 relative);
  * MXFP8 SwiGLU rows h (MXFP4 layers), element by element: within one E4M3 step
    of the oracle's value at its magnitude (2^-3 |h|, or 2^-9 of the block scale
    for values below the E4M3 normal range), scale codes equal except where the
    block's amax lies within 1e-4 (relative) of a power of two.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import moe as om

GAP_EXACT = 1e-6
TOL_Y = 2e-2          # of RMS(y_oracle)
TOL_Y_REL = 2.0 ** -8  # of |y_oracle|: the BF16 rounding of y itself, twice
TOL_W = 1e-5


def output_score(y_gpu, y_oracle) -> float:
    """TOL_Y x the largest ratio of |y_gpu - y_oracle| to its element's bound
    TOL_Y RMS(y_oracle) + TOL_Y_REL |y_oracle|: below TOL_Y exactly when every element
    is within its bound (0 for an exact match, also when the oracle is all zero)."""
    yg = np.asarray(y_gpu, dtype=np.float64)
    yo = np.asarray(y_oracle, dtype=np.float64)
    d = np.abs(yg - yo)
    rms = float(np.sqrt(np.mean(yo ** 2)))
    bound = TOL_Y * rms + TOL_Y_REL * np.abs(yo)
    if np.any((bound == 0) & (d > 0)):
        return float("inf")
    ratio = np.divide(d, bound, out=np.zeros_like(d), where=bound > 0)
    return TOL_Y * float(ratio.max()) if ratio.size else 0.0


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a BF16/fp32 tensor (any device)."""
    return t.detach().to("cpu").to(torch.float64).numpy()


def _bf16_bits_to_f64(u16: np.ndarray) -> np.ndarray:
    """Exact float64 values of BF16 bit patterns (uint16)."""
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _mx_roundtrip_expert(job):
    """Worker: the oracle's MX round trip (element format 'e2m1' or 'e4m3') of one
    expert's three BF16 matrices (uint16 bit patterns); float32 holds every result
    exactly."""
    from oracle import mx as omx
    fmt, mats = job
    return tuple(omx.mx_roundtrip(_bf16_bits_to_f64(m), fmt).astype(np.float32) for m in mats)


def _u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def oracle_pool(n: int | None = None):
    """A spawn-started process pool for the oracle's per-expert work (safe after CUDA is initialised)."""
    import multiprocessing as mp
    import os
    n = n or max(1, min(16, len(os.sched_getaffinity(0))))
    return mp.get_context("spawn").Pool(n)


class LayerExperts(om.ExpertSource):
    """Oracle expert source reading one expert at a time from the generator's tensors.

    mx_from_bf16: the routed experts are the oracle's own MXFP4 (mx_fmt 'e2m1') or
    MXFP8 ('e4m3') quantisation of the BF16 draw; mx_q: given MXFP4 (packed) or
    MXFP8 tensors. With a process pool and the list of experts the comparison needs
    (in the order the oracle visits them), that quantisation runs in the pool,
    a batch of experts at a time; the oracle itself is unchanged.
    """

    def __init__(self, layer: dict, mx_q: dict | None = None, mx_from_bf16: bool = False, pool=None,
                 needed=None, mx_fmt: str = "e2m1"):
        S = layer["sh_w1"].shape[0]
        E = layer["w1"].shape[0]
        self._layer = layer
        self._pool = pool
        self._needed = [int(e) for e in needed] if needed is not None else None
        self._cache = {}
        self._fmt = mx_fmt
        if mx_from_bf16:
            from oracle import mx as omx
            if pool is None or needed is None:
                rt = lambda w: omx.mx_roundtrip(f64(w), mx_fmt)
                routed = lambda e: (rt(layer["w1"][e]), rt(layer["w3"][e]), rt(layer["w2"][e]))
            else:
                routed = self._pooled_mx
            is_mx = True
        elif mx_q is None:
            routed = lambda e: (f64(layer["w1"][e]), f64(layer["w3"][e]), f64(layer["w2"][e]))
            is_mx = False
        else:
            from oracle import mx as omx
            fp8 = mx_q["w1"].shape[-1] == layer["w1"].shape[-1]
            dqf = omx.dequantize_mxfp8 if fp8 else omx.dequantize_mxfp4_packed
            dq = lambda q, s, e: dqf(q[e].cpu().numpy(), s[e].cpu().numpy())
            routed = lambda e: (dq(mx_q["w1"], mx_q["s1"], e), dq(mx_q["w3"], mx_q["s3"], e),
                                dq(mx_q["w2"], mx_q["s2"], e))
            is_mx = True
        shared = lambda j: (f64(layer["sh_w1"][j]), f64(layer["sh_w3"][j]), f64(layer["sh_w2"][j]))
        super().__init__(routed, shared, E, S, routed_is_mx=is_mx)

    def _pooled_mx(self, e):
        if e not in self._cache:
            self._cache.clear()
            pos = self._needed.index(e) if e in self._needed else None
            batch = self._needed[pos:pos + 2 * self._pool._processes] if pos is not None else [e]
            lay = self._layer
            jobs = [(self._fmt, (_u16(lay["w1"][b]), _u16(lay["w3"][b]), _u16(lay["w2"][b]))) for b in batch]
            for b, mats in zip(batch, self._pool.map(_mx_roundtrip_expert, jobs)):
                self._cache[b] = mats
        return tuple(m.astype(np.float64) for m in self._cache[e])


def covering_tokens(idx, n_routed, n_shared=0, block=32):
    """Tokens whose rows reach every `block`-row slice of every expert group.

    The grouped GEMMs lay each expert's rows out in ascending (token, slot) order
    and cut them into token tiles of at most 256 rows, loaded in 32-row boxes; a
    mistake in one tile's or one box's offsets shows only in the tokens whose rows
    fall inside it. Covering every 32-row slice of every routed group (and of each
    shared group, whose rows are the tokens in order) therefore exercises every
    token tile, every box, and, because each compared row spans the whole hidden
    and expert width, every weight tile. Greedy: the first token of each slice not
    yet reached. Returns sorted token indices.
    """
    idx = np.asarray(idx, dtype=np.int64)
    T, k = idx.shape
    flat = idx.reshape(-1)
    order = np.argsort(flat, kind="stable")
    counts = np.bincount(flat, minlength=n_routed)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    row_in_group = np.empty(T * k, dtype=np.int64)
    row_in_group[order] = np.arange(T * k) - offsets[flat[order]]
    nblk = (T + block - 1) // block
    pair = flat * nblk + row_in_group // block          # routed (expert, slice)
    tok_pairs = pair.reshape(T, k)
    covered = set()
    chosen = []
    first_slot = {}
    for s in order:                                     # ascending rows inside each expert
        first_slot.setdefault(int(pair[s]), int(s))
    for p in sorted(first_slot):
        if p in covered:
            continue
        t = first_slot[p] // k
        chosen.append(t)
        covered.update(int(q) for q in tok_pairs[t])
    if n_shared > 0:
        have = {t // block for t in chosen}
        chosen.extend(b * block for b in range(nblk) if b not in have)
    return np.array(sorted(set(chosen)), dtype=np.int64)


def oracle_route(layer, k, rs, tokens=None):
    x = layer["x"] if tokens is None else layer["x"][tokens]
    bias = None if layer.get("bias") is None else f64(layer["bias"])
    return om.route(f64(x), f64(layer["wg"]), k, rs, bias=bias)


def compare_layer(layer, tokens, y_gpu, idx_gpu, w_gpu, k, rs, limit, mx_q=None, mx_from_bf16=False, pool=None,
                  mx_fmt="e2m1"):
    """Compare GPU rows (for `tokens`) with the oracle; returns a report dict, asserts the bars.

    With mx_q (packed MXFP4 tensors) or mx_from_bf16 the routed experts are MXFP4 and
    the oracle mirrors the MXFP8 activation quantisation. `pool` (oracle_pool())
    spreads the oracle's MXFP4 quantisation of the experts over processes."""
    tokens = np.asarray(tokens)
    x = f64(layer["x"][torch.as_tensor(tokens, device=layer["x"].device)])
    wg = f64(layer["wg"])
    bias = None if layer.get("bias") is None else f64(layer["bias"])
    r = om.route(x, wg, k, rs, bias=bias)
    idx_g = np.asarray(idx_gpu, dtype=np.int64)
    sure = r.gap > GAP_EXACT
    mism = np.where(sure & np.any(idx_g != r.idx, axis=1))[0]
    assert len(mism) == 0, f"top-k differs on {len(mism)} tokens with gap > 1e-6, e.g. token {tokens[mism[:3]]}: " \
                           f"gpu {idx_g[mism[:1]]} oracle {r.idx[mism[:1]]} gap {r.gap[mism[:1]]}"
    # outputs: use the GPU's selection where the oracle's gap is within the tie band
    override = np.where(sure[:, None], r.idx, idx_g)
    ex = LayerExperts(layer, mx_q, mx_from_bf16, pool=pool, needed=np.unique(override), mx_fmt=mx_fmt)
    res = om.moe_forward(x, wg, ex, k, rs, limit, bias=bias, idx_override=override)
    w_or = res.route.w
    dw = np.abs(np.asarray(w_gpu, dtype=np.float64) - w_or).max()
    assert dw <= TOL_W, f"routing weights differ by {dw}"
    yg = np.asarray(y_gpu, dtype=np.float64)
    yo = res.y
    rms = float(np.sqrt(np.mean(yo ** 2)))
    err = float(np.abs(yg - yo).max())
    assert np.all(np.isfinite(yg)), "non-finite GPU output"
    score = output_score(yg, yo)
    assert score < TOL_Y, f"max|dy| = {err:.3e} (RMS {rms:.3e}): {score / TOL_Y:.3f} of the element bound"
    return dict(max_abs_err=err, rms=rms, rel=score, rel_rms=err / rms if rms > 0 else 0.0,
                near_ties=int((~sure).sum()), max_dw=float(dw), tokens=len(tokens))


def check_nan_token(layer, lay, T, bad, k, E, rs, limit, mx_q=None):
    """Forward T tokens of lay["x"] with token `bad` set to NaN; assert the NaN stays
    in that token and the others still match the oracle."""
    import routed_expert_ffn_sqrtsoftplus_b200 as moe
    x = lay["x"][:T].clone()
    x[bad] = float("nan")
    y, idx, w = layer.forward_with_routing(x)
    torch.cuda.synchronize()
    # the token's scores are NaN: placeholder experts 0..k-1, NaN weights, NaN row,
    # and the status word says so; the other tokens are computed as usual
    assert layer.status() == moe.MOE_ERR_DEVICE
    assert layer.status() == moe.MOE_OK
    idx_np, w_np, y_np = idx.cpu().numpy(), w.cpu().numpy(), y.float().cpu().numpy()
    assert np.all((idx_np >= 0) & (idx_np < E))
    assert list(idx_np[bad]) == list(range(k))
    assert np.all(np.isnan(w_np[bad])) and np.all(np.isnan(y_np[bad]))
    keep = np.setdiff1d(np.arange(T), [bad])
    rep = compare_layer(dict(lay, x=x), keep, y_np[keep], idx_np[keep], w_np[keep], k, rs,
                          limit, mx_q=mx_q)
    assert rep["rel"] < TOL_Y
    # the next forward on finite input is clean
    layer.forward(lay["x"][:T].contiguous())
    torch.cuda.synchronize()
    assert layer.status() == moe.MOE_OK


def compare_hashed(layer, tokens, ids, table, y_gpu, idx_gpu, w_gpu, k, rs, limit, mx_q=None):
    """Hash-routed layer: indices equal to the table rows of the ids, weights and
    outputs against the oracle's moe_forward_hashed on the same tokens."""
    tokens = np.asarray(tokens)
    x = f64(layer["x"][torch.as_tensor(tokens, device=layer["x"].device)])
    bias = None if layer.get("bias") is None else f64(layer["bias"])
    tab = table.cpu().numpy().astype(np.int64)
    ids_np = np.asarray(ids, dtype=np.int64)[tokens]
    assert np.array_equal(np.asarray(idx_gpu, dtype=np.int64), tab[ids_np]), "selection differs from the table"
    ex = LayerExperts(layer, mx_q)
    res = om.moe_forward_hashed(x, f64(layer["wg"]), ex, tab, ids_np, rs, limit, bias=bias)
    dw = float(np.abs(np.asarray(w_gpu, dtype=np.float64) - res.route.w).max())
    assert dw <= TOL_W, f"routing weights differ by {dw}"
    yg = np.asarray(y_gpu, dtype=np.float64)
    rms = float(np.sqrt(np.mean(res.y ** 2)))
    err = float(np.abs(yg - res.y).max())
    score = output_score(yg, res.y)
    assert np.all(np.isfinite(yg)) and score < TOL_Y, \
        f"max|dy| = {err:.3e} (RMS {rms:.3e}): {score / TOL_Y:.3f} of the element bound"
    return dict(max_abs_err=err, rms=rms, rel=score, rel_rms=err / rms if rms > 0 else 0.0, max_dw=dw,
                tokens=len(tokens))
