"""GPU parity of hash-routed layers (MAX DeepseekV41Config num_hash_layers):
experts from a vocabulary table row per token id, weights the normalised
sqrtsoftplus scores, through the C ABI against the oracle's moe_forward_hashed."""
import numpy as np
import pytest
import torch

import routed_expert_ffn_sqrtsoftplus_b200 as moe
from routed_expert_ffn_sqrtsoftplus_b200 import build, synth

import parity

pytestmark = pytest.mark.gpu

WL = synth.WORKLOADS["tiny"]
VOCAB = 1000


@pytest.fixture(scope="module")
def hashed(cuda_device):
    build.build()
    lay = synth.make_layer(WL.with_tokens(700), device="cpu")
    lay = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in lay.items()}
    table = synth.make_hash_table(WL, VOCAB, device=cuda_device)
    ids = synth.make_token_ids(WL, VOCAB, device=cuda_device, T=700)
    layer = moe.MoELayer.from_layer(lay, top_k=WL.k, max_tokens=700)
    layer.set_hash_table(table)
    yield lay, table, ids, layer
    layer.close()


def _run(layer, x, ids):
    T = x.shape[0]
    idx = torch.empty((T, WL.k), dtype=torch.int32, device=x.device)
    w = torch.empty((T, WL.k), dtype=torch.float32, device=x.device)
    y = layer.forward_hashed(x, ids, topk_idx=idx, topk_w=w)
    torch.cuda.synchronize()
    return y, idx, w


@pytest.mark.parametrize("T", [1, 17, 64, 300, 700])
def test_hashed_layer_parity(hashed, T):
    lay, table, ids, layer = hashed
    x = lay["x"][:T].contiguous()
    y, idx, w = _run(layer, x, ids[:T].contiguous())
    assert layer.status() == moe.MOE_OK
    rep = parity.compare_hashed(dict(lay, x=x), np.arange(T), ids[:T].cpu().numpy(), table, y.float().cpu().numpy(),
                                idx.cpu().numpy(), w.cpu().numpy(), WL.k, WL.route_scale, WL.swiglu_limit)
    assert rep["rel"] < parity.TOL_Y


def test_hashed_layer_with_mxfp4_experts(cuda_device):
    from oracle import mx as omx
    lay = synth.make_layer(WL.with_tokens(64), device="cpu")
    q = {}
    for n, sname in (("w1", "s1"), ("w3", "s3"), ("w2", "s2")):
        a, b = omx.quantize_mxfp4_packed(parity.f64(lay[n]))
        q[n], q[sname] = torch.from_numpy(np.ascontiguousarray(a)), torch.from_numpy(np.ascontiguousarray(b))
    lay = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in lay.items()}
    q = {k: v.to(cuda_device) for k, v in q.items()}
    table = synth.make_hash_table(WL, VOCAB, device=cuda_device)
    ids = synth.make_token_ids(WL, VOCAB, device=cuda_device, T=64)
    layer = moe.MoELayer.from_layer(lay, top_k=WL.k, max_tokens=64, mx=q)
    try:
        layer.set_hash_table(table)
        for T in (5, 64):
            x = lay["x"][:T].contiguous()
            y, idx, w = _run(layer, x, ids[:T].contiguous())
            assert layer.status() == moe.MOE_OK
            rep = parity.compare_hashed(dict(lay, x=x), np.arange(T), ids[:T].cpu().numpy(), table,
                                        y.float().cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy(), WL.k,
                                        WL.route_scale, WL.swiglu_limit, mx_q=q)
            assert rep["rel"] < parity.TOL_Y
    finally:
        layer.close()


def test_hash_table_is_checked(hashed, cuda_device):
    lay, table, ids, layer = hashed
    bad = table.clone()
    bad[17, 3] = bad[17, 1]                  # an expert twice in one row
    with pytest.raises(moe.MoEError) as ei:
        layer.set_hash_table(bad)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
    bad = table.clone()
    bad[400, 0] = WL.E                       # outside [0, E)
    with pytest.raises(moe.MoEError) as ei:
        layer.set_hash_table(bad)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
    # the layer keeps its earlier table
    x = lay["x"][:8].contiguous()
    _, idx, _ = _run(layer, x, ids[:8].contiguous())
    assert torch.equal(idx, table[ids[:8].long()])


def test_out_of_range_id_is_contained(hashed):
    lay, table, ids, layer = hashed
    T = 40
    x = lay["x"][:T].contiguous()
    bad_ids = ids[:T].clone()
    bad_ids[9] = VOCAB + 5
    y, idx, w = _run(layer, x, bad_ids)
    assert layer.status() == moe.MOE_ERR_DEVICE
    assert idx[9].tolist() == list(range(WL.k)) and bool(torch.isnan(w[9]).all())
    assert bool(torch.isnan(y[9].float()).all())
    keep = np.setdiff1d(np.arange(T), [9])
    rep = parity.compare_hashed(dict(lay, x=x), keep, bad_ids.cpu().numpy(), table, y.float().cpu().numpy()[keep],
                                idx.cpu().numpy()[keep], w.cpu().numpy()[keep], WL.k, WL.route_scale,
                                WL.swiglu_limit)
    assert rep["rel"] < parity.TOL_Y


def test_forward_hashed_needs_a_table(cuda_device):
    lay = synth.make_layer(WL.with_tokens(8), device="cpu")
    lay = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in lay.items()}
    layer = moe.MoELayer.from_layer(lay, top_k=WL.k, max_tokens=8)
    try:
        with pytest.raises(moe.MoEError) as ei:
            layer.forward_hashed(lay["x"], torch.zeros(8, dtype=torch.int32, device=cuda_device))
        assert ei.value.status == moe.MOE_ERR_INVALID_ARG
    finally:
        layer.close()


@pytest.mark.slow
def test_flash_decode_hashed_full(cuda_device):
    """The Flash decode shape (T=32) with a hash table over the full 129,280-token vocabulary."""
    build.build()
    wl = synth.WORKLOADS["flash_decode"]
    lay = synth.make_layer(wl, device=cuda_device)
    table = synth.make_hash_table(wl, device=cuda_device)
    ids = synth.make_token_ids(wl, device=cuda_device)
    layer = moe.MoELayer.from_layer(lay, top_k=wl.k, max_tokens=wl.T)
    try:
        layer.set_hash_table(table)
        y, idx, w = _run(layer, lay["x"], ids)
        assert layer.status() == moe.MOE_OK
        rep = parity.compare_hashed(lay, np.arange(wl.T), ids.cpu().numpy(), table, y.float().cpu().numpy(),
                                    idx.cpu().numpy(), w.cpu().numpy(), wl.k, wl.route_scale, wl.swiglu_limit)
        print(rep)
        assert rep["rel"] < parity.TOL_Y
    finally:
        layer.close()
        del lay
        torch.cuda.empty_cache()
