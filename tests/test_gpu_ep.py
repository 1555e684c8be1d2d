"""GPU parity of expert-parallel partial outputs (moe_create_ep / moe_forward_partial)
on one GPU: two handles holding complementary windows of the routed experts
stand in for two ranks in one process (no collective; ExpertParallelLayer's
exchange is covered on CPU by tests/test_ep_dist.py). Each partial output is
compared with the oracle's moe_forward_partial, their sum with the whole layer."""
import numpy as np
import pytest
import torch

import routed_expert_ffn_sqrtsoftplus_b200 as moe
from routed_expert_ffn_sqrtsoftplus_b200 import build, synth
from oracle import moe as om
from oracle import mx as omx

import parity

pytestmark = pytest.mark.gpu

WL = synth.WORKLOADS["tiny"]


def _mxq(lay, fmt):
    quant = omx.quantize_mxfp8 if fmt == "mxfp8" else omx.quantize_mxfp4_packed
    out = {}
    for n, sname in (("w1", "s1"), ("w3", "s3"), ("w2", "s2")):
        q, sc = quant(parity.f64(lay[n]))
        out[n], out[sname] = torch.from_numpy(np.ascontiguousarray(q)), torch.from_numpy(np.ascontiguousarray(sc))
    return out


@pytest.mark.parametrize("mx", [False, "mxfp4", "mxfp8"], ids=["bf16", "mxfp4", "mxfp8"])
@pytest.mark.parametrize("split", [16, 11])
def test_partial_outputs_of_two_windows(cuda_device, mx, split):
    build.build()
    Tmax = 300
    lay = synth.make_layer(WL.with_tokens(Tmax), device="cpu")
    q = _mxq(lay, mx) if mx else None
    lay = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in lay.items()}
    if q is not None:
        q = {k: v.to(cuda_device) for k, v in q.items()}
    wins = [(0, split), (split, WL.E - split)]
    layers = [moe.MoELayer.from_layer(lay, top_k=WL.k, max_tokens=Tmax, mx=q, expert_window=w, with_shared=(i == 0))
              for i, w in enumerate(wins)]
    try:
        ex = parity.LayerExperts(lay, mx_q=q)
        wg = parity.f64(lay["wg"])
        for T in (5, 64, 300):
            x = lay["x"][:T].contiguous()
            parts = [L.forward_partial(x) for L in layers]
            torch.cuda.synchronize()
            for L in layers:
                assert L.status() == moe.MOE_OK
            xf = parity.f64(x)
            full = om.moe_forward(xf, wg, ex, WL.k, WL.route_scale, WL.swiglu_limit)
            rms = float(np.sqrt(np.mean(full.y ** 2)))
            # near-tie tokens may legitimately route differently; none in this draw
            assert np.all(full.route.gap > parity.GAP_EXACT)
            for i, ((b, c), p) in enumerate(zip(wins, parts)):
                ref = om.moe_forward_partial(xf, wg, ex, WL.k, WL.route_scale, WL.swiglu_limit, b, b + c,
                                             include_shared=(i == 0))
                score = parity.output_score(p.double().cpu().numpy(), ref)
                assert score < parity.TOL_Y, f"window {b}..{b + c}, T={T}: {score / parity.TOL_Y:.3f} of the bound"
            y = (parts[0] + parts[1]).double().cpu().numpy()
            assert parity.output_score(y, full.y) < parity.TOL_Y
    finally:
        for L in layers:
            L.close()


def test_whole_layer_partial_is_the_forward_in_fp32(cuda_device):
    build.build()
    lay = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v)
           for k, v in synth.make_layer(WL.with_tokens(64)).items()}
    layer = moe.MoELayer.from_layer(lay, top_k=WL.k, max_tokens=64)
    try:
        x = lay["x"]
        y16 = layer.forward(x).float()
        y32 = layer.forward_partial(x)
        torch.cuda.synchronize()
        # the BF16 output is the fp32 sum rounded once
        assert torch.equal(y32.to(torch.bfloat16).float(), y16)
    finally:
        layer.close()


def test_window_handle_refuses_the_whole_forward(cuda_device):
    build.build()
    lay = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v)
           for k, v in synth.make_layer(WL.with_tokens(8)).items()}
    layer = moe.MoELayer.from_layer(lay, top_k=WL.k, max_tokens=8, expert_window=(4, 8))
    try:
        with pytest.raises(moe.MoEError) as ei:
            layer.forward(lay["x"])
        assert ei.value.status == moe.MOE_ERR_INVALID_ARG
        with pytest.raises(ValueError):
            moe.MoELayer.from_layer(lay, top_k=WL.k, max_tokens=8, expert_window=(30, 8))   # past the last expert
    finally:
        layer.close()
