"""Parity helpers: run the oracle on the same seeded inputs and compare.

Tolerances (fixed before any kernel ran):
  * routing: for every token whose oracle gap s_(k) - s_(k+1) exceeds 1e-6 the
    selected experts must equal the oracle's, in the same descending order;
    tokens at or below that gap may pick differently, and their oracle output
    is recomputed with the GPU's choice;
  * routing weights: |w_gpu - w_oracle| <= 1e-5 (fp32 rounding of an fp64 value);
  * layer output: max |y_gpu - y_oracle| <= 2e-2 * RMS(y_oracle) over the compared
    rows (BF16 rounding of h and y, fp32 accumulation);
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
TOL_Y = 2e-2
TOL_W = 1e-5


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a BF16/fp32 tensor (any device)."""
    return t.detach().to("cpu").to(torch.float64).numpy()


class LayerExperts(om.ExpertSource):
    """Oracle expert source reading one expert at a time from the generator's tensors."""

    def __init__(self, layer: dict, mx_q: dict | None = None, mx_from_bf16: bool = False):
        S = layer["sh_w1"].shape[0]
        E = layer["w1"].shape[0]
        if mx_from_bf16:
            # quantise each routed expert with the oracle's own MXFP4 codec
            from oracle import mx as omx
            rt = lambda w: omx.mx_roundtrip(f64(w), "e2m1")
            routed = lambda e: (rt(layer["w1"][e]), rt(layer["w3"][e]), rt(layer["w2"][e]))
            is_mx = True
        elif mx_q is None:
            routed = lambda e: (f64(layer["w1"][e]), f64(layer["w3"][e]), f64(layer["w2"][e]))
            is_mx = False
        else:
            from oracle import mx as omx
            dq = lambda q, s, e: omx.dequantize_mxfp4_packed(q[e].cpu().numpy(), s[e].cpu().numpy())
            routed = lambda e: (dq(mx_q["w1"], mx_q["s1"], e), dq(mx_q["w3"], mx_q["s3"], e),
                                dq(mx_q["w2"], mx_q["s2"], e))
            is_mx = True
        shared = lambda j: (f64(layer["sh_w1"][j]), f64(layer["sh_w3"][j]), f64(layer["sh_w2"][j]))
        super().__init__(routed, shared, E, S, routed_is_mx=is_mx)


def oracle_route(layer, k, rs, tokens=None):
    x = layer["x"] if tokens is None else layer["x"][tokens]
    bias = None if layer.get("bias") is None else f64(layer["bias"])
    return om.route(f64(x), f64(layer["wg"]), k, rs, bias=bias)


def compare_layer(layer, tokens, y_gpu, idx_gpu, w_gpu, k, rs, limit, mx_q=None, mx_from_bf16=False):
    """Compare GPU rows (for `tokens`) with the oracle; returns a report dict, asserts the bars.

    With mx_q (packed MXFP4 tensors) or mx_from_bf16 the routed experts are MXFP4 and
    the oracle mirrors the MXFP8 activation quantisation."""
    tokens = np.asarray(tokens)
    x = f64(layer["x"][torch.as_tensor(tokens, device=layer["x"].device)])
    wg = f64(layer["wg"])
    bias = None if layer.get("bias") is None else f64(layer["bias"])
    ex = LayerExperts(layer, mx_q, mx_from_bf16)
    r = om.route(x, wg, k, rs, bias=bias)
    idx_g = np.asarray(idx_gpu, dtype=np.int64)
    sure = r.gap > GAP_EXACT
    mism = np.where(sure & np.any(idx_g != r.idx, axis=1))[0]
    assert len(mism) == 0, f"top-k differs on {len(mism)} tokens with gap > 1e-6, e.g. token {tokens[mism[:3]]}: " \
                           f"gpu {idx_g[mism[:1]]} oracle {r.idx[mism[:1]]} gap {r.gap[mism[:1]]}"
    # outputs: use the GPU's selection where the oracle's gap is within the tie band
    override = np.where(sure[:, None], r.idx, idx_g)
    res = om.moe_forward(x, wg, ex, k, rs, limit, bias=bias, idx_override=override)
    w_or = res.route.w
    dw = np.abs(np.asarray(w_gpu, dtype=np.float64) - w_or).max()
    assert dw <= TOL_W, f"routing weights differ by {dw}"
    yg = np.asarray(y_gpu, dtype=np.float64)
    yo = res.y
    rms = float(np.sqrt(np.mean(yo ** 2)))
    err = float(np.abs(yg - yo).max())
    assert np.all(np.isfinite(yg)), "non-finite GPU output"
    assert err <= TOL_Y * rms, f"max|dy| = {err:.3e} > {TOL_Y} * RMS {rms:.3e}"
    return dict(max_abs_err=err, rms=rms, rel=err / rms, near_ties=int((~sure).sum()), max_dw=float(dw))
