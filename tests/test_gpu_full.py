"""GPU parity at the full workload sizes, in the configuration bench.py times
(one layer created with max_tokens = T, one forward over all T tokens).

Routing is checked for every token against the oracle's float64 router; the
layer output is checked on all tokens (decode) or on a seeded sample of tokens
the oracle evaluates one expert at a time (prefill, V4-Pro)."""
import gc

import numpy as np
import pytest
import torch

import routed_expert_ffn_sqrtsoftplus_b200 as moe
from routed_expert_ffn_sqrtsoftplus_b200 import build, synth

import parity

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _free():
    gc.collect()
    torch.cuda.empty_cache()


def _run_workload(name, cuda_device):
    build.build()
    wl = synth.WORKLOADS[name]
    lay = synth.make_layer(wl, device=cuda_device)
    layer = moe.MoELayer.from_layer(lay, top_k=wl.k, max_tokens=wl.T, route_scale=wl.route_scale,
                                    swiglu_limit=wl.swiglu_limit)
    try:
        y, idx, w = layer.forward_with_routing(lay["x"])
        torch.cuda.synchronize()
        assert layer.status() == moe.MOE_OK
        idx_np, w_np = idx.cpu().numpy(), w.cpu().numpy()
        y_cpu = y.float().cpu().numpy()
        assert np.all(np.isfinite(y_cpu))
        # routing of every token
        r = parity.oracle_route(lay, wl.k, wl.route_scale)
        sure = r.gap > parity.GAP_EXACT
        bad = np.where(sure & np.any(idx_np != r.idx, axis=1))[0]
        assert len(bad) == 0, f"{len(bad)} tokens route differently (gap > 1e-6), first {bad[:5]}"
        ok = sure
        assert np.abs(w_np[ok] - r.w[ok]).max() <= parity.TOL_W
        # the permutation covers every (token, slot) exactly once
        G = wl.E + wl.n_shared
        cnt = layer.inspect(moe.BUF_COUNTS, torch.empty(G, dtype=torch.int32, device=cuda_device)).cpu().numpy()
        assert cnt[:wl.E].sum() == wl.T * wl.k and np.all(cnt[wl.E:] == wl.T)
        assert np.array_equal(cnt[:wl.E], np.bincount(idx_np.ravel(), minlength=wl.E))
        # outputs: every token at decode; otherwise a sample reaching every 32-row
        # slice of every expert group (every token tile, B box and weight tile)
        toks = np.arange(wl.T) if wl.T <= 32 else parity.covering_tokens(idx_np, wl.E, wl.n_shared)
        rep = parity.compare_layer(lay, toks, y_cpu[toks], idx_np[toks], w_np[toks], wl.k, wl.route_scale,
                                   wl.swiglu_limit)
        rep["near_tie_tokens_all"] = int((~sure).sum())
        print(name, rep)
        return rep, cnt
    finally:
        layer.close()
        del lay
        _free()


def test_flash_decode_full(cuda_device):
    rep, _ = _run_workload("flash_decode", cuda_device)
    assert rep["rel"] < parity.TOL_Y


def test_flash_prefill_full(cuda_device):
    rep, cnt = _run_workload("flash_prefill", cuda_device)
    assert rep["rel"] < parity.TOL_Y


def test_pro_skewed_full(cuda_device):
    rep, cnt = _run_workload("pro_skewed", cuda_device)
    assert rep["rel"] < parity.TOL_Y
    # Zipf-biased routing: the most popular expert takes a large share of the tokens
    assert cnt[:384].max() > 0.5 * synth.WORKLOADS["pro_skewed"].T
