"""A seeded sweep of layer configurations against the oracle, through the C ABI:
BF16, MXFP4 and MXFP8 routed experts; 0 to 2 shared experts; top-k 1 to 16;
8 to 512 routed experts; hidden 128 to 2048 (multiples of 128, some not of 256);
expert width 128 to 512;
uniform and skewed routers (a per-expert bias, so that a few experts take several
token tiles and many get a handful of rows); and token counts from one to many
tokens per expert, so that each case runs the routing, permutation, tile-list,
GEMM and combine variants its shape selects. The cases are drawn once from a
fixed seed and do not change between runs."""
import numpy as np
import pytest
import torch

import routed_expert_ffn_sqrtsoftplus_b200 as moe
from routed_expert_ffn_sqrtsoftplus_b200 import build, synth
from oracle import mx as omx

import parity

pytestmark = pytest.mark.gpu


def _cases(n=24, seed=20241203):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        E = int(rng.choice([8, 12, 16, 24, 32, 48, 64]))
        k = int(rng.integers(1, min(8, E) + 1))
        H = int(rng.choice([128, 256, 384, 512]))
        I = int(rng.choice([128, 256]))
        S = int(rng.integers(0, 3))
        fmt = str(rng.choice(["bf16", "mxfp4", "mxfp8"]))
        skew = bool(rng.integers(0, 2))
        Ts = sorted({int(rng.integers(1, 33)), int(rng.integers(33, 129)), int(rng.integers(129, 401))})
        out.append((f"c{i}-{fmt}-E{E}k{k}H{H}I{I}S{S}{'-skew' if skew else ''}", E, k, H, I, S, fmt, skew, Ts))
    return out


def _large_cases(n=12, seed=20241204):
    """Larger layers: many experts, wider k and widths, up to 1200 tokens (several
    permutation chunks, both many-token tile widths, the thin-tile split)."""
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        fmt = str(rng.choice(["bf16", "mxfp4", "mxfp8"]))
        # block-scaled layers kept smaller: the oracle's codec quantises them on the host
        E = int(rng.choice([128, 256, 384, 512] if fmt == "bf16" else [128, 256]))
        k = int(rng.choice([4, 6, 8, 12, 16]))
        H = int(rng.choice([512, 768, 1024, 2048] if fmt == "bf16" else [512, 768, 1024]))
        I = int(rng.choice([256, 512] if fmt == "bf16" else [256]))
        S = int(rng.integers(0, 3))
        skew = bool(rng.integers(0, 2))
        Ts = sorted({int(rng.integers(1, 33)), int(rng.integers(200, 601)), int(rng.integers(601, 1201))})
        out.append((f"L{i}-{fmt}-E{E}k{k}H{H}I{I}S{S}{'-skew' if skew else ''}", E, k, H, I, S, fmt, skew, Ts))
    return out


CASES = _cases() + _large_cases()


def _quantised(lay, fmt):
    quant = omx.quantize_mxfp8 if fmt == "mxfp8" else omx.quantize_mxfp4_packed
    q = {}
    for n, sname in (("w1", "s1"), ("w3", "s3"), ("w2", "s2")):
        a, sc = quant(parity.f64(lay[n]))
        q[n], q[sname] = torch.from_numpy(np.ascontiguousarray(a)), torch.from_numpy(np.ascontiguousarray(sc))
    return q


@pytest.mark.parametrize("name,E,k,H,I,S,fmt,skew,Ts", CASES, ids=[c[0] for c in CASES])
def test_sweep_case(cuda_device, name, E, k, H, I, S, fmt, skew, Ts):
    build.build()
    tag = name.split("-")[0]
    wl = synth.Workload(name, T=0, H=H, I=I, E=E, k=k, n_shared=S,
                        seed=(3000 if tag[0] == "c" else 3100) + int(tag[1:]))
    Tmax = max(Ts)
    lay = synth.make_layer(wl.with_tokens(Tmax), device="cpu")
    if skew:
        # the first experts of a seeded order take most tokens (bias 2 ln(1/rank))
        order = torch.randperm(E, generator=torch.Generator().manual_seed(wl.seed))
        rank = torch.empty(E, dtype=torch.float64)
        rank[order] = torch.arange(1, E + 1, dtype=torch.float64)
        lay["bias"] = (2.0 * torch.log(1.0 / rank)).to(torch.float32)
    q = _quantised(lay, fmt) if fmt != "bf16" else None
    lay = {n: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for n, v in lay.items()}
    if q is not None:
        q = {n: v.to(cuda_device) for n, v in q.items()}
    layer = moe.MoELayer.from_layer(lay, top_k=k, max_tokens=Tmax, mx=q)
    try:
        for T in Ts:
            x = lay["x"][:T].contiguous()
            y, idx, w = layer.forward_with_routing(x)
            torch.cuda.synchronize()
            assert layer.status() == moe.MOE_OK, f"T={T}"
            rep = parity.compare_layer(dict(lay, x=x), np.arange(T), y.float().cpu().numpy(), idx.cpu().numpy(),
                                       w.cpu().numpy(), k, wl.route_scale, wl.swiglu_limit, mx_q=q)
            assert rep["rel"] < parity.TOL_Y, f"T={T}: {rep}"
    finally:
        layer.close()
