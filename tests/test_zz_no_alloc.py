"""moe_route_noalloc: routing for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc at all (their device memory belongs to a
host framework's pool, or their loop forbids allocation once running); for
them the library offers routing whose one scratch buffer is a fixed array
inside the library. This test calls that entry point through the C ABI and
checks it against the float64 oracle's routing and against the routing
moe_forward returns for the same tokens, on calls in a row (each with a
different token count, so each runs over what the one before left in the
shared array). It sits in its own file, collected last.
"""
import ctypes

import numpy as np

import pytest
import torch

import routed_expert_ffn_sqrtsoftplus_b200 as moe
from routed_expert_ffn_sqrtsoftplus_b200 import build, synth

import parity

pytestmark = pytest.mark.gpu

WL = synth.WORKLOADS["tiny"]
MAX_LOGITS = 1 << 20   # MOE_NOALLOC_MAX_LOGITS in include/moe.h


def _route_noalloc(x, wg, bias, k, rs):
    T, H = x.shape
    E = wg.shape[0]
    idx = torch.full((T, k), -1, dtype=torch.int32, device=x.device)
    w = torch.full((T, k), float("nan"), dtype=torch.float32, device=x.device)
    st = moe.lib().moe_route_noalloc(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(wg.data_ptr()),
                                     None if bias is None else ctypes.c_void_p(bias.data_ptr()),
                                     T, H, E, k, ctypes.c_float(rs), ctypes.c_void_p(idx.data_ptr()),
                                     ctypes.c_void_p(w.data_ptr()),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, idx, w


def _check_against_oracle(lay, T, idx, w, k, rs):
    """Routing parity bar: indices equal to the float64 oracle's wherever its gap
    exceeds 1e-6, weights within float32 rounding."""
    r = parity.oracle_route(dict(lay, x=lay["x"][:T]), k, rs)
    sure = r.gap > parity.GAP_EXACT
    idx_np, w_np = idx.cpu().numpy(), w.cpu().numpy()
    assert not np.any(sure & np.any(idx_np != r.idx, axis=1))
    assert np.abs(w_np[sure] - r.w[sure]).max() <= parity.TOL_W
    return sure


def test_route_noalloc_matches_forward(cuda_device):
    build.build()
    Tmax = 2000
    lay = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v)
           for k, v in synth.make_layer(WL.with_tokens(Tmax)).items()}
    layer = moe.MoELayer.from_layer(lay, top_k=WL.k, max_tokens=Tmax)
    try:
        # calls in a row over the one shared array: the second smaller than the
        # first, the third above 1024 tokens (one warp per token in the top-k)
        for T in (96, 23, Tmax):
            x = lay["x"][:T].contiguous()
            _, idx_ref, w_ref = layer.forward_with_routing(x)
            st, idx, w = _route_noalloc(x, lay["wg"], lay["bias"], WL.k, WL.route_scale)
            torch.cuda.synchronize()
            assert st == moe.MOE_OK
            sure = torch.as_tensor(_check_against_oracle(lay, T, idx, w, WL.k, WL.route_scale), device=idx.device)
            assert torch.equal(idx[sure], idx_ref[sure])
            assert (w - w_ref).abs().max().item() <= parity.TOL_W
    finally:
        layer.close()


def test_route_noalloc_nan_token_gets_placeholders(cuda_device):
    build.build()
    lay = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v)
           for k, v in synth.make_layer(WL.with_tokens(40)).items()}
    x = lay["x"].clone()
    x[7] = float("nan")
    st, idx, w = _route_noalloc(x, lay["wg"], None, WL.k, WL.route_scale)
    torch.cuda.synchronize()
    assert st == moe.MOE_OK
    assert idx[7].tolist() == list(range(WL.k)) and bool(torch.isnan(w[7]).all())
    keep = [t for t in range(40) if t != 7]
    assert bool(((idx >= 0) & (idx < WL.E)).all())
    r = parity.oracle_route(dict(lay, x=lay["x"][keep]), WL.k, WL.route_scale)
    sure = r.gap > parity.GAP_EXACT
    assert not np.any(sure & np.any(idx[keep].cpu().numpy() != r.idx, axis=1))


def test_route_noalloc_with_bias_and_limit(cuda_device):
    build.build()
    wl = synth.Workload("zipf_tiny", T=40, H=512, I=256, E=32, zipf_bias=True, seed=77)
    lay = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in synth.make_layer(wl).items()}
    layer = moe.MoELayer.from_layer(lay, top_k=wl.k, max_tokens=wl.T)
    try:
        _, idx_ref, w_ref = layer.forward_with_routing(lay["x"])
        st, idx, w = _route_noalloc(lay["x"], lay["wg"], lay["bias"], wl.k, wl.route_scale)
        torch.cuda.synchronize()
        assert st == moe.MOE_OK
        assert torch.equal(idx, idx_ref) and (w - w_ref).abs().max().item() <= parity.TOL_W
    finally:
        layer.close()
    # beyond the fixed scratch: refused, nothing written
    T_big = MAX_LOGITS // wl.E + 1
    x_big = torch.zeros((T_big, wl.H), dtype=torch.bfloat16, device=cuda_device)
    st, idx, _ = _route_noalloc(x_big, lay["wg"], None, wl.k, wl.route_scale)
    torch.cuda.synchronize()
    assert st == moe.MOE_ERR_UNSUPPORTED
    assert bool((idx == -1).all())
