"""GPU parity of the MXFP4 routed-expert path (E2M1 weights, E8M0 scales per 32,
MXFP8 activations) against the oracle in MX mirror mode, through the C ABI."""
import numpy as np
import pytest
import torch

import routed_expert_ffn_sqrtsoftplus_b200 as moe
from routed_expert_ffn_sqrtsoftplus_b200 import build, synth
from oracle import mx as omx

import parity

pytestmark = pytest.mark.gpu

WL = synth.WORKLOADS["tiny"]


def _oracle_quantised(lay):
    """MXFP4 tensors produced by the oracle's codec from the BF16 draw (CPU)."""
    out = {}
    for n, sname in (("w1", "s1"), ("w3", "s3"), ("w2", "s2")):
        q, sc = omx.quantize_mxfp4_packed(parity.f64(lay[n]))
        out[n] = torch.from_numpy(np.ascontiguousarray(q))
        out[sname] = torch.from_numpy(np.ascontiguousarray(sc))
    return out


@pytest.fixture(scope="module")
def tiny_mx(cuda_device):
    build.build()
    lay = synth.make_layer(WL.with_tokens(400), device="cpu")
    mxq_cpu = _oracle_quantised(lay)
    lay = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in lay.items()}
    mxq = {k: v.to(cuda_device) for k, v in mxq_cpu.items()}
    layer = moe.MoELayer.from_layer(lay, top_k=WL.k, max_tokens=400, mx=mxq)
    yield lay, mxq, layer
    layer.close()


@pytest.mark.parametrize("T", [16, 1, 5, 33, 64, 300])
def test_tiny_mx_layer_parity(tiny_mx, T):
    lay, mxq, layer = tiny_mx
    x = lay["x"][:T].contiguous()
    y, idx, w = layer.forward_with_routing(x)
    torch.cuda.synchronize()
    assert layer.status() == moe.MOE_OK
    rep = parity.compare_layer(dict(lay, x=x), np.arange(T), y.float().cpu().numpy(), idx.cpu().numpy(),
                               w.cpu().numpy(), WL.k, WL.route_scale, WL.swiglu_limit, mx_q=mxq)
    assert rep["rel"] < parity.TOL_Y


def test_mx_activation_codes_bitexact(tiny_mx):
    """The MXFP8 codes of the routed token rows equal the oracle's quantisation of x."""
    lay, mxq, layer = tiny_mx
    T = 64
    x = lay["x"][:T].contiguous()
    layer.forward(x)
    xq = layer.inspect(moe.BUF_XQ, torch.empty((T * WL.k, WL.H), dtype=torch.uint8, device=x.device))
    perm = layer.inspect(moe.BUF_PERM, torch.empty(T * WL.k, dtype=torch.int32, device=x.device))
    torch.cuda.synchronize()
    codes_ref, _ = omx.quantize_mx(parity.f64(x), "e4m3")
    rows = perm.cpu().numpy() // WL.k
    got = xq.cpu().numpy()
    # compare decoded values (the two encodings of zero are the same value)
    assert np.array_equal(omx.decode_e4m3(got), omx.decode_e4m3(codes_ref[rows]))


def test_mx_deterministic(tiny_mx):
    lay, _, layer = tiny_mx
    x = lay["x"][:300].contiguous()
    y1 = layer.forward(x).clone()
    y2 = layer.forward(x)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_mx_rejects_nan_scale(cuda_device):
    build.build()
    lay = synth.make_layer(WL.with_tokens(8), device="cpu")
    mxq = _oracle_quantised(lay)
    mxq["s3"][2, 5, 1] = 0xFF
    lay = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in lay.items()}
    mxq = {k: v.to(cuda_device) for k, v in mxq.items()}
    with pytest.raises(moe.MoEError) as ei:
        moe.MoELayer.from_layer(lay, top_k=WL.k, max_tokens=8, mx=mxq)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG


@pytest.mark.slow
@pytest.mark.parametrize("name,n_sample", [("flash_mxfp4_decode", 6), ("flash_mxfp4_prefill", 6)])
def test_flash_mxfp4_full(cuda_device, name, n_sample):
    build.build()
    wl = synth.WORKLOADS[name]
    lay = synth.make_layer(wl, device=cuda_device)
    mxq = {}
    for n, sname in (("w1", "s1"), ("w3", "s3"), ("w2", "s2")):
        mxq[n], mxq[sname] = moe.quantize_mxfp4(lay[n])
    layer = moe.MoELayer.from_layer(lay, top_k=wl.k, max_tokens=wl.T, mx=mxq)
    try:
        y, idx, w = layer.forward_with_routing(lay["x"])
        torch.cuda.synchronize()
        assert layer.status() == moe.MOE_OK
        toks = np.arange(wl.T) if n_sample >= wl.T else \
            np.sort(np.random.default_rng(wl.seed).choice(wl.T, n_sample, replace=False))
        y_np = y.float().cpu().numpy()
        assert np.all(np.isfinite(y_np))
        # the oracle quantises the BF16 draw itself (its codec matches moe_quantize_mxfp4 bit for bit)
        rep = parity.compare_layer(lay, toks, y_np[toks], idx.cpu().numpy()[toks], w.cpu().numpy()[toks], wl.k,
                                   wl.route_scale, wl.swiglu_limit, mx_from_bf16=True)
        print(name, rep)
        assert rep["rel"] < parity.TOL_Y
    finally:
        layer.close()
        del lay, mxq
        torch.cuda.empty_cache()
