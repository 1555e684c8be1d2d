"""GPU parity of the MXFP4 routed-expert path (E2M1 weights, E8M0 scales per 32,
MXFP8 activations) against the oracle in MX mirror mode, through the C ABI."""
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


@pytest.mark.parametrize("T", [300])
def test_tiny_mx_layer_parity_hot_experts(tiny_mx, cuda_device, T):
    """A router bias of +6 on experts 0 and 1 sends every token to both: each of
    them gets several full 96-token MX tiles and a partial one, which the tile list
    keeps next to the full ones (their token-tile ids, scale atoms and h rows)."""
    lay, mxq, _ = tiny_mx
    bias = torch.zeros(WL.E, dtype=torch.float32, device=cuda_device)
    bias[:2] = 6.0
    hot = dict(lay, bias=bias)
    layer = moe.MoELayer.from_layer(hot, top_k=WL.k, max_tokens=400, mx=mxq)
    try:
        x = lay["x"][:T].contiguous()
        y, idx, w = layer.forward_with_routing(x)
        torch.cuda.synchronize()
        assert layer.status() == moe.MOE_OK
        cnt = np.bincount(idx.cpu().numpy().ravel(), minlength=WL.E)
        assert cnt[0] == T and cnt[1] == T
        rep = parity.compare_layer(dict(hot, x=x), np.arange(T), y.float().cpu().numpy(), idx.cpu().numpy(),
                                   w.cpu().numpy(), WL.k, WL.route_scale, WL.swiglu_limit, mx_q=mxq)
        assert rep["rel"] < parity.TOL_Y
    finally:
        layer.close()


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


def _hq_values(hq, sf, cnt, T, k, E, I):
    """Decode the MXFP8 h rows the gate/up epilogue wrote (codes + scale atoms, the
    layout include/moe.h gives for MOE_BUF_HQ / MOE_BUF_HQ_SCALES)."""
    bn = 32 if T <= 32 else (96 if T * k >= 24 * E else 64)
    off = np.concatenate([[0], np.cumsum(cnt)])
    ntb = np.concatenate([[0], np.cumsum((cnt + bn - 1) // bn)])
    R = T * k
    g = np.searchsorted(off, np.arange(R), side="right") - 1
    j = np.arange(R) - off[g]
    nt, n = ntb[g] + j // bn, j % bn
    b = np.arange(I // 32)
    addr = (nt[:, None] * (I // 128) + b[None, :] // 4) * 512 + (n[:, None] % 32) * 16 + (n[:, None] // 32) * 4 \
        + b[None, :] % 4
    codes = sf[addr]
    vals = omx.dequantize_mx(hq, codes, "e4m3")
    return vals, codes


@pytest.mark.parametrize("T", [16, 64, 300])
def test_mx_swiglu_rows_match_oracle(tiny_mx, T):
    """The MXFP8 h rows (E4M3 codes and E8M0 scales) that the MX gate/up epilogue
    writes, element by element, against the oracle's h of the same expert on the
    same MXFP8 token: within one E4M3 step at the value's magnitude, scale codes
    equal wherever the block's amax is not within 1e-4 of a power of two."""
    lay, mxq, layer = tiny_mx
    x = lay["x"][:T].contiguous()
    _, idx, _ = layer.forward_with_routing(x)
    R = T * WL.k
    dev = x.device
    hq = layer.inspect(moe.BUF_HQ, torch.empty((R, WL.I), dtype=torch.uint8, device=dev))
    sf = layer.inspect(moe.BUF_HQ_SCALES, torch.empty(_hq_scale_cap(), dtype=torch.uint8, device=dev))
    perm = layer.inspect(moe.BUF_PERM, torch.empty(R, dtype=torch.int32, device=dev))
    cnt = layer.inspect(moe.BUF_COUNTS, torch.empty(WL.E + WL.n_shared, dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    assert layer.status() == moe.MOE_OK
    cnt = cnt.cpu().numpy()[:WL.E].astype(np.int64)
    vals, codes = _hq_values(hq.cpu().numpy(), sf.cpu().numpy(), cnt, T, WL.k, WL.E, WL.I)
    perm = perm.cpu().numpy()
    idx = idx.cpu().numpy().reshape(-1)
    xf = parity.f64(x)
    ex = parity.LayerExperts(lay, mx_q=mxq)
    flips = 0
    for e in range(WL.E):
        rows = np.nonzero(idx[perm] == e)[0]
        if len(rows) == 0:
            continue
        _, h_or = om.expert_forward(xf[perm[rows] // WL.k], *ex.routed(e), WL.swiglu_limit, mx_act=True)
        q_or, sc_or = omx.quantize_mx(h_or, "e4m3")
        amax = np.abs(h_or.reshape(len(rows), -1, 32)).max(axis=-1)
        l2 = np.log2(np.where(amax > 0, amax, 1.0))
        near_pow2 = np.abs(l2 - np.round(l2)) < 1.5e-4
        assert np.all((codes[rows] == sc_or) | near_pow2), f"expert {e}: scale codes differ"
        X = np.repeat(omx.decode_e8m0(sc_or), 32, axis=-1)
        bound = 2.0 ** -3 * np.abs(h_or) + 2.0 ** -8 * X
        err = np.abs(vals[rows] - h_or)
        assert np.all(err <= bound), f"expert {e}: max err / bound {np.max(err / bound)}"
        flips += int(np.sum(omx.decode_e4m3(hq.cpu().numpy()[rows]) * X != omx.dequantize_mx(q_or, sc_or, "e4m3")))
    print(f"T={T}: element codes differing from the oracle's (RNE neighbours): {flips}")


def _hq_scale_cap():
    """Bytes of the h scale atoms a layer with max_tokens 400 holds (tiny shape)."""
    return (WL.E + (400 * WL.k + 31) // 32) * (WL.I // 128) * 512


@pytest.mark.parametrize("T,bad", [(16, 3), (64, 40)])
def test_mx_nan_token_is_contained(tiny_mx, T, bad):
    lay, mxq, layer = tiny_mx
    parity.check_nan_token(layer, lay, T, bad, WL.k, WL.E, WL.route_scale, WL.swiglu_limit, mx_q=mxq)


@pytest.mark.parametrize("T", [5, 40, 300])
def test_mx_poisoned_workspace_gives_the_same_bits(tiny_mx, T):
    lay, _, layer = tiny_mx
    x = lay["x"][:T].contiguous()
    y1 = layer.forward(x).clone()
    torch.cuda.synchronize()
    layer.fill_workspace(0xFF)
    y2 = layer.forward(x)
    torch.cuda.synchronize()
    assert layer.status() == moe.MOE_OK
    assert torch.equal(y1, y2)


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
@pytest.mark.parametrize("name", ["flash_mxfp4_decode", "flash_mxfp4_prefill"])
def test_flash_mxfp4_full(cuda_device, name):
    """Full-size MXFP4 layers. Outputs compared on every token at decode, and at
    prefill on a sample that reaches every 32-row slice of every expert group
    (every token tile and weight tile of every expert that has rows); the oracle
    quantises the BF16 draw itself, spread over a spawn-started process pool."""
    build.build()
    wl = synth.WORKLOADS[name]
    pool = parity.oracle_pool()
    lay = synth.make_layer(wl, device=cuda_device)
    mxq = {}
    for n, sname in (("w1", "s1"), ("w3", "s3"), ("w2", "s2")):
        mxq[n], mxq[sname] = moe.quantize_mxfp4(lay[n])
    layer = moe.MoELayer.from_layer(lay, top_k=wl.k, max_tokens=wl.T, mx=mxq)
    try:
        y, idx, w = layer.forward_with_routing(lay["x"])
        torch.cuda.synchronize()
        assert layer.status() == moe.MOE_OK
        idx_np = idx.cpu().numpy()
        toks = np.arange(wl.T) if wl.T <= 32 else parity.covering_tokens(idx_np, wl.E, wl.n_shared)
        y_np = y.float().cpu().numpy()
        assert np.all(np.isfinite(y_np))
        # routing of every token against the oracle's float64 router
        r = parity.oracle_route(lay, wl.k, wl.route_scale)
        sure = r.gap > parity.GAP_EXACT
        assert not np.any(sure & np.any(idx_np != r.idx, axis=1))
        del mxq
        rep = parity.compare_layer(lay, toks, y_np[toks], idx_np[toks], w.cpu().numpy()[toks], wl.k,
                                   wl.route_scale, wl.swiglu_limit, mx_from_bf16=True, pool=pool)
        print(name, rep)
        assert rep["rel"] < parity.TOL_Y
    finally:
        pool.terminate()
        layer.close()
        del lay
        torch.cuda.empty_cache()
