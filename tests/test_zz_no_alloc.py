"""moe_route_noalloc: routing for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc at all (their device memory belongs to a
host framework's pool, or their loop forbids allocation once running); for
them the library offers routing whose one scratch buffer is a fixed array
inside the library. This test calls that entry point through the C ABI and
checks it against the routing moe_forward returns for the same tokens, on two
calls in a row (the second with a different token count, so it runs over what
the first left in the shared array). It sits in its own file, collected last.
"""
import ctypes

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


def test_route_noalloc_matches_forward(cuda_device):
    build.build()
    lay = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v)
           for k, v in synth.make_layer(WL.with_tokens(96)).items()}
    layer = moe.MoELayer.from_layer(lay, top_k=WL.k, max_tokens=96)
    try:
        for T in (96, 23):                       # two calls in a row, the second smaller
            x = lay["x"][:T].contiguous()
            _, idx_ref, w_ref = layer.forward_with_routing(x)
            st, idx, w = _route_noalloc(x, lay["wg"], lay["bias"], WL.k, WL.route_scale)
            torch.cuda.synchronize()
            assert st == moe.MOE_OK
            assert torch.equal(idx, idx_ref)
            assert (w - w_ref).abs().max().item() <= parity.TOL_W
    finally:
        layer.close()


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
