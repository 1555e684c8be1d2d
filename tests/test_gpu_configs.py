"""GPU parity of layer configurations moe_create accepts beyond the pages' shape,
each at few tokens (T <= 32: sliced router, 32-row tiles), a middle count (one
token tile per expert) and many tokens per expert (tensor-core router, the
widest tiles), through the C ABI against the oracle:

  * swiglu_limit 0 (the layer output is exactly zero) and infinity (no clamp);
  * top_k = n_routed (every expert selected);
  * 0, 2 and 4 shared experts (4 is the most moe_create accepts), with BF16,
    MXFP4 and MXFP8 routed experts (the block-scaled paths run the shared experts
    separately: split-K at few tokens, their own tile lists otherwise);
  * top_k = 1;
  * the widest hidden and expert widths accepted (16384);
  * 512 routed experts with top-32 (the widest top-k instantiation, and more
    slots than one permutation chunk);
  * MXFP4 and MXFP8 routed experts with hidden % 256 != 0 (128-row W2 tiles in
    the block-scaled down GEMM).
"""
import math

import numpy as np
import pytest
import torch

import routed_expert_ffn_sqrtsoftplus_b200 as moe
from routed_expert_ffn_sqrtsoftplus_b200 import build, synth
from oracle import mx as omx

import parity

pytestmark = pytest.mark.gpu


def _oracle_mxfp4(lay):
    """MXFP4 bytes of the routed experts, quantised by the oracle's codec on the host."""
    out = {}
    for n, sname in (("w1", "s1"), ("w3", "s3"), ("w2", "s2")):
        q, sc = omx.quantize_mxfp4_packed(parity.f64(lay[n]))
        out[n] = torch.from_numpy(np.ascontiguousarray(q))
        out[sname] = torch.from_numpy(np.ascontiguousarray(sc))
    return out


def _oracle_mxfp8(lay):
    """MXFP8 codes and scales of the routed experts from the oracle's codec (host)."""
    out = {}
    for n, sname in (("w1", "s1"), ("w3", "s3"), ("w2", "s2")):
        q, sc = omx.quantize_mxfp8(parity.f64(lay[n]))
        out[n] = torch.from_numpy(np.ascontiguousarray(q))
        out[sname] = torch.from_numpy(np.ascontiguousarray(sc))
    return out


def _check(wl, Ts, cuda_device, mx=False, sample=None):
    """mx: False (BF16 experts), True or "mxfp4", or "mxfp8". sample: compare at most
    this many tokens, spread over the batch (all of them when None)."""
    build.build()
    Tmax = max(Ts)
    lay = synth.make_layer(wl.with_tokens(Tmax), device="cpu")
    mxq = None
    if mx:
        mxq = _oracle_mxfp8(lay) if mx == "mxfp8" else _oracle_mxfp4(lay)
    lay = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in lay.items()}
    if mxq is not None:
        mxq = {k: v.to(cuda_device) for k, v in mxq.items()}
    layer = moe.MoELayer.from_layer(lay, top_k=wl.k, max_tokens=Tmax, route_scale=wl.route_scale,
                                    swiglu_limit=wl.swiglu_limit, mx=mxq)
    reps = []
    try:
        for T in Ts:
            x = lay["x"][:T].contiguous()
            y, idx, w = layer.forward_with_routing(x)
            torch.cuda.synchronize()
            assert layer.status() == moe.MOE_OK
            toks = np.arange(T) if sample is None or T <= sample else np.unique(np.linspace(0, T - 1, sample).astype(int))
            rep = parity.compare_layer(dict(lay, x=x), toks, y.float().cpu().numpy()[toks], idx.cpu().numpy()[toks],
                                       w.cpu().numpy()[toks], wl.k, wl.route_scale, wl.swiglu_limit, mx_q=mxq)
            assert rep["rel"] < parity.TOL_Y
            reps.append((T, rep, y))
    finally:
        layer.close()
    return reps


BASE = synth.Workload("cfg", T=0, H=256, I=128, E=16, k=4, seed=2001)


MX = pytest.mark.parametrize("mx", [False, "mxfp4", "mxfp8"], ids=["bf16", "mxfp4", "mxfp8"])


@MX
def test_swiglu_limit_zero_gives_zero(cuda_device, mx):
    wl = synth.Workload("cfg_l0", T=0, H=256, I=128, E=16, k=4, swiglu_limit=0.0, seed=2002)
    for T, rep, y in _check(wl, [5, 40, 300], cuda_device, mx):
        assert rep["rms"] == 0.0 and rep["max_abs_err"] == 0.0
        assert not bool(torch.any(y != 0))


@MX
def test_swiglu_limit_infinite(cuda_device, mx):
    wl = synth.Workload("cfg_linf", T=0, H=256, I=128, E=16, k=4, swiglu_limit=math.inf, seed=2003)
    _check(wl, [5, 40, 300], cuda_device, mx)


def test_every_expert_selected(cuda_device):
    wl = synth.Workload("cfg_kE", T=0, H=128, I=128, E=8, k=8, seed=2004)
    for T, rep, _ in _check(wl, [3, 20, 40, 300], cuda_device):
        assert rep["near_ties"] == 0


@pytest.mark.parametrize("S", [0, 2, 4])
@MX
def test_shared_expert_count(cuda_device, S, mx):
    wl = synth.Workload(f"cfg_s{S}", T=0, H=256, I=128, E=16, k=4, n_shared=S, seed=2005 + S)
    _check(wl, [5, 32, 40, 300], cuda_device, mx)


def test_512_experts_top32(cuda_device):
    wl = synth.Workload("cfg_e512", T=0, H=128, I=128, E=512, k=32, seed=2008)
    _check(wl, [5, 40, 400], cuda_device)


@pytest.mark.parametrize("mx", ["mxfp4", "mxfp8"])
def test_block_scaled_hidden_not_multiple_of_256(cuda_device, mx):
    wl = synth.Workload("cfg_h384", T=0, H=384, I=256, E=16, k=4, seed=2009)
    _check(wl, [5, 40, 300], cuda_device, mx=mx)


@MX
def test_top1(cuda_device, mx):
    wl = synth.Workload("cfg_k1", T=0, H=256, I=128, E=16, k=1, seed=2010)
    _check(wl, [5, 40, 300], cuda_device, mx)


def test_widest_hidden(cuda_device):
    wl = synth.Workload("cfg_h16k", T=0, H=16384, I=128, E=8, k=2, seed=2011)
    _check(wl, [3, 40, 200], cuda_device)


def test_widest_expert(cuda_device):
    wl = synth.Workload("cfg_i16k", T=0, H=256, I=16384, E=8, k=2, seed=2012)
    _check(wl, [3, 40, 200], cuda_device)
