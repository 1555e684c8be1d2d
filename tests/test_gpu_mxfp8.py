"""GPU parity of the MXFP8 routed-expert path (E4M3 weights, E8M0 scales per 32,
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


def _oracle_mxfp8(lay):
    """MXFP8 codes and scales of the routed experts from the oracle's codec (host)."""
    out = {}
    for n, sname in (("w1", "s1"), ("w3", "s3"), ("w2", "s2")):
        q, sc = omx.quantize_mxfp8(parity.f64(lay[n]))
        out[n] = torch.from_numpy(np.ascontiguousarray(q))
        out[sname] = torch.from_numpy(np.ascontiguousarray(sc))
    return out


@pytest.fixture(scope="module")
def tiny_f8(cuda_device):
    build.build()
    lay = synth.make_layer(WL.with_tokens(400), device="cpu")
    q = _oracle_mxfp8(lay)
    lay = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in lay.items()}
    q = {k: v.to(cuda_device) for k, v in q.items()}
    layer = moe.MoELayer.from_layer(lay, top_k=WL.k, max_tokens=400, mx=q)
    yield lay, q, layer
    layer.close()


@pytest.mark.parametrize("T", [16, 1, 5, 33, 64, 300])
def test_tiny_mxfp8_layer_parity(tiny_f8, T):
    lay, q, layer = tiny_f8
    x = lay["x"][:T].contiguous()
    y, idx, w = layer.forward_with_routing(x)
    torch.cuda.synchronize()
    assert layer.status() == moe.MOE_OK
    rep = parity.compare_layer(dict(lay, x=x), np.arange(T), y.float().cpu().numpy(), idx.cpu().numpy(),
                               w.cpu().numpy(), WL.k, WL.route_scale, WL.swiglu_limit, mx_q=q)
    assert rep["rel"] < parity.TOL_Y


def test_tiny_mxfp8_layer_parity_hot_experts(tiny_f8, cuda_device):
    """Every token sent to experts 0 and 1 (router bias +6): several full 96-token
    tiles and a partial one for each of them, with E4M3 weights."""
    lay, q, _ = tiny_f8
    T = 300
    bias = torch.zeros(WL.E, dtype=torch.float32, device=cuda_device)
    bias[:2] = 6.0
    hot = dict(lay, bias=bias)
    layer = moe.MoELayer.from_layer(hot, top_k=WL.k, max_tokens=400, mx=q)
    try:
        x = lay["x"][:T].contiguous()
        y, idx, w = layer.forward_with_routing(x)
        torch.cuda.synchronize()
        assert layer.status() == moe.MOE_OK
        cnt = np.bincount(idx.cpu().numpy().ravel(), minlength=WL.E)
        assert cnt[0] == T and cnt[1] == T
        rep = parity.compare_layer(dict(hot, x=x), np.arange(T), y.float().cpu().numpy(), idx.cpu().numpy(),
                                   w.cpu().numpy(), WL.k, WL.route_scale, WL.swiglu_limit, mx_q=q)
        assert rep["rel"] < parity.TOL_Y
    finally:
        layer.close()


def test_mxfp8_layer_follows_the_mxfp8_oracle(tiny_f8):
    """The GPU output is closer to the oracle's MXFP8 layer than to its BF16 layer on
    the same draw: the path computes the MXFP8 semantics, not another format's."""
    from oracle import moe as om
    lay, q, layer = tiny_f8
    T = 64
    x = lay["x"][:T].contiguous()
    y, idx, _ = layer.forward_with_routing(x)
    torch.cuda.synchronize()
    xf, wg = parity.f64(x), parity.f64(lay["wg"])
    ov = dict(idx_override=idx.cpu().numpy())
    y_mx = om.moe_forward(xf, wg, parity.LayerExperts(lay, mx_q=q), WL.k, WL.route_scale, WL.swiglu_limit, **ov).y
    y_bf = om.moe_forward(xf, wg, parity.LayerExperts(lay), WL.k, WL.route_scale, WL.swiglu_limit, **ov).y
    yg = y.double().cpu().numpy()
    d_mx, d_bf = np.abs(yg - y_mx).max(), np.abs(yg - y_bf).max()
    print(f"max |y - oracle MXFP8| = {d_mx:.3e}, max |y - oracle BF16| = {d_bf:.3e}")
    assert d_mx < 0.5 * d_bf


def test_quantize_mxfp8_bitexact(cuda_device):
    g = torch.Generator().manual_seed(13)
    w = (torch.randn((48, 512), generator=g) * 0.03).to(torch.bfloat16)
    w[3, :32] = 0                                  # all-zero block
    w[4, 32:64] = 1000.0                           # amax 1000: scale 2^1, elements saturate at 448
    w[4, 40] = 1e-30                               # far below the block's smallest E4M3 step
    w[6, :32] = torch.finfo(torch.bfloat16).tiny   # smallest normal BF16
    w[7, 64:96] = torch.tensor([1.0 + 2 ** -4, 1.0 + 3 * 2 ** -4, 448.0, -3.0] * 8)   # E4M3 ties at scale 1
    q, s = moe.quantize_mxfp8(w.to(cuda_device))
    torch.cuda.synchronize()
    q_ref, s_ref = omx.quantize_mxfp8(parity.f64(w))
    assert np.array_equal(s.cpu().numpy(), s_ref)
    # compare values (the two encodings of zero decode alike)
    assert np.array_equal(omx.decode_e4m3(q.cpu().numpy()), omx.decode_e4m3(q_ref))


@pytest.mark.slow
@pytest.mark.parametrize("name", ["flash_mxfp8_decode", "flash_mxfp8_prefill"])
def test_flash_mxfp8_full(cuda_device, name):
    """Full-size MXFP8 layers: every token at decode, the tile-covering sample at
    prefill; the oracle quantises the BF16 draw itself in a process pool."""
    build.build()
    wl = synth.WORKLOADS[name]
    pool = parity.oracle_pool()
    lay = synth.make_layer(wl, device=cuda_device)
    q = {}
    for n, sname in (("w1", "s1"), ("w3", "s3"), ("w2", "s2")):
        q[n], q[sname] = moe.quantize_mxfp8(lay[n])
    layer = moe.MoELayer.from_layer(lay, top_k=wl.k, max_tokens=wl.T, mx=q)
    del q
    try:
        y, idx, w = layer.forward_with_routing(lay["x"])
        torch.cuda.synchronize()
        assert layer.status() == moe.MOE_OK
        idx_np = idx.cpu().numpy()
        r = parity.oracle_route(lay, wl.k, wl.route_scale)
        sure = r.gap > parity.GAP_EXACT
        assert not np.any(sure & np.any(idx_np != r.idx, axis=1))
        toks = np.arange(wl.T) if wl.T <= 32 else parity.covering_tokens(idx_np, wl.E, wl.n_shared)
        y_np = y.float().cpu().numpy()
        rep = parity.compare_layer(lay, toks, y_np[toks], idx_np[toks], w.cpu().numpy()[toks], wl.k,
                                   wl.route_scale, wl.swiglu_limit, mx_from_bf16=True, pool=pool, mx_fmt="e4m3")
        print(name, rep)
        assert rep["rel"] < parity.TOL_Y
    finally:
        pool.terminate()
        layer.close()
        del lay
        torch.cuda.empty_cache()
