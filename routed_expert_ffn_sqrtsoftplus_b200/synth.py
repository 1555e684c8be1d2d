"""Seeded synthetic workloads for the MoE layer (inputs only: no layer arithmetic here).

Both the CUDA path's tests/bench and the oracle draw their inputs from this
module; it computes nothing the layer computes. Every draw is N(0, 1) in fp32
from a seeded ``torch.Generator``, multiplied by the stated standard deviation
and rounded to BF16 (round-to-nearest-even). "N(0, 1/n)" in the workload
descriptions means variance 1/n, so a router logit x . Wg_e is about N(0, 1).

Workloads (shapes from the DeepSeek V4.1 inference/config.json and the
DeepSeek-V4-Pro config paragraph; distributions as stated per workload):
  tiny                T=64,   H=512,  I=256,  32 routed + 1 shared, top-6
  flash_decode        T=32,   H=5120, I=2304, 384 + 1, top-6
  flash_prefill       T=8192, same layer as flash_decode
  flash_mxfp4_decode  T=16,   same layer, routed experts to be stored as MXFP4
  flash_mxfp4_prefill T=4096, same
  flash_mxfp8_decode  T=32,   same layer, routed experts to be stored as MXFP8
                      (E4M3 + E8M0 per 32)
  flash_mxfp8_prefill T=4096, same (the MXFP4 prefill batch)
  pro_skewed          T=2048, H=7168, I=3072, 384 + 1, top-6, with a Zipf
                      per-expert logit bias b_e = 2 ln(1/rank_e) over a seeded
                      random expert permutation (a few experts get most tokens)
  dspark              T=256,  H=5120, I=2304, 128 routed + 1 shared, top-3
                      (the drafter's expert count and top-k from the config;
                      its widths are not printed, the main layer's are assumed)
All use route_scale 1.5 and swiglu_limit 10. The MXFP4 and MXFP8 workloads draw
BF16 weights exactly like flash_decode; quantising them is the consumer's job.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    I: int
    E: int
    n_shared: int = 1
    k: int = 6
    route_scale: float = 1.5
    swiglu_limit: float = 10.0
    expert_dtype: str = "bf16"          # "bf16" | "mxfp4" | "mxfp8" (routed experts)
    zipf_bias: bool = False
    seed: int = 1000

    def with_tokens(self, T: int) -> "Workload":
        return replace(self, T=T)

    @property
    def weight_bytes_bf16_per_expert(self) -> int:
        return 3 * self.H * self.I * 2


WORKLOADS = {
    "tiny": Workload("tiny", T=64, H=512, I=256, E=32, seed=1000),
    "flash_decode": Workload("flash_decode", T=32, H=5120, I=2304, E=384, seed=1001),
    "flash_prefill": Workload("flash_prefill", T=8192, H=5120, I=2304, E=384, seed=1002),
    "flash_mxfp4_decode": Workload("flash_mxfp4_decode", T=16, H=5120, I=2304, E=384,
                                   expert_dtype="mxfp4", seed=1003),
    "flash_mxfp4_prefill": Workload("flash_mxfp4_prefill", T=4096, H=5120, I=2304, E=384,
                                    expert_dtype="mxfp4", seed=1003),
    "flash_mxfp8_decode": Workload("flash_mxfp8_decode", T=32, H=5120, I=2304, E=384,
                                   expert_dtype="mxfp8", seed=1006),
    "flash_mxfp8_prefill": Workload("flash_mxfp8_prefill", T=4096, H=5120, I=2304, E=384,
                                    expert_dtype="mxfp8", seed=1006),
    "pro_skewed": Workload("pro_skewed", T=2048, H=7168, I=3072, E=384, zipf_bias=True, seed=1004),
    "dspark": Workload("dspark", T=256, H=5120, I=2304, E=128, k=3, seed=1005),
}


def _normal_bf16(shape, std, gen, device):
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    t.mul_(std)
    return t.to(torch.bfloat16)


def make_tokens(wl: Workload, device="cpu", T: Optional[int] = None, seed: Optional[int] = None):
    """x ~ N(0, 1), BF16 [T, H], from its own seeded stream."""
    T = wl.T if T is None else T
    gen = torch.Generator(device=device)
    gen.manual_seed((wl.seed if seed is None else seed) * 7919 + 17)
    return _normal_bf16((T, wl.H), 1.0, gen, device)


def make_router(wl: Workload, device="cpu", seed: Optional[int] = None):
    """Wg ~ N(0, 1/H) BF16 [E, H]; bias fp32 [E] (Zipf workloads) or None."""
    gen = torch.Generator(device=device)
    gen.manual_seed((wl.seed if seed is None else seed) * 7919 + 29)
    wg = _normal_bf16((wl.E, wl.H), 1.0 / math.sqrt(wl.H), gen, device)
    bias = None
    if wl.zipf_bias:
        pgen = torch.Generator(device="cpu")
        pgen.manual_seed((wl.seed if seed is None else seed) * 7919 + 31)
        rank = torch.randperm(wl.E, generator=pgen).to(torch.float64) + 1.0   # 1-based ranks
        bias = (2.0 * torch.log(1.0 / rank)).to(torch.float32).to(device)
    return wg, bias


def make_experts(wl: Workload, device="cpu", seed: Optional[int] = None):
    """Routed W1, W3 [E, I, H] ~ N(0, 1/H), W2 [E, H, I] ~ N(0, 1/I); shared likewise.

    Generated one expert at a time so the fp32 scratch stays one expert large.
    """
    E, S, H, I = wl.E, wl.n_shared, wl.H, wl.I
    gen = torch.Generator(device=device)
    gen.manual_seed((wl.seed if seed is None else seed) * 7919 + 43)
    w1 = torch.empty((E, I, H), dtype=torch.bfloat16, device=device)
    w3 = torch.empty((E, I, H), dtype=torch.bfloat16, device=device)
    w2 = torch.empty((E, H, I), dtype=torch.bfloat16, device=device)
    s1 = torch.empty((S, I, H), dtype=torch.bfloat16, device=device)
    s3 = torch.empty((S, I, H), dtype=torch.bfloat16, device=device)
    s2 = torch.empty((S, H, I), dtype=torch.bfloat16, device=device)
    sh, si = 1.0 / math.sqrt(H), 1.0 / math.sqrt(I)
    for dst1, dst3, dst2, n in ((w1, w3, w2, E), (s1, s3, s2, S)):
        for e in range(n):
            dst1[e].copy_(_normal_bf16((I, H), sh, gen, device))
            dst3[e].copy_(_normal_bf16((I, H), sh, gen, device))
            dst2[e].copy_(_normal_bf16((H, I), si, gen, device))
    return dict(w1=w1, w3=w3, w2=w2, sh_w1=s1, sh_w3=s3, sh_w2=s2)


VOCAB = 129280   # DeepSeek V4.1 vocabulary (MAX DeepseekV41Config vocab_size)


def make_hash_table(wl: Workload, vocab: int = VOCAB, device="cpu", seed: Optional[int] = None):
    """Vocabulary table of a hash-routed layer: int32 [vocab, k], each row k distinct
    experts (the k largest of E seeded uniform draws), from its own seeded stream."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed((wl.seed if seed is None else seed) * 7919 + 53)
    out = torch.empty((vocab, wl.k), dtype=torch.int32)
    for v0 in range(0, vocab, 16384):
        v1 = min(vocab, v0 + 16384)
        out[v0:v1] = torch.rand((v1 - v0, wl.E), generator=gen).topk(wl.k, dim=1).indices.to(torch.int32)
    return out.to(device)


def make_token_ids(wl: Workload, vocab: int = VOCAB, device="cpu", T: Optional[int] = None,
                   seed: Optional[int] = None):
    """Token ids uniform over the vocabulary, int32 [T], from their own seeded stream."""
    T = wl.T if T is None else T
    gen = torch.Generator(device="cpu")
    gen.manual_seed((wl.seed if seed is None else seed) * 7919 + 59)
    return torch.randint(0, vocab, (T,), generator=gen, dtype=torch.int64).to(torch.int32).to(device)


def make_layer(wl: Workload, device="cpu", T: Optional[int] = None, seed: Optional[int] = None):
    """All inputs of one layer invocation: x, wg, bias and the expert weights."""
    x = make_tokens(wl, device, T=T, seed=seed)
    wg, bias = make_router(wl, device, seed=seed)
    d = make_experts(wl, device, seed=seed)
    d.update(x=x, wg=wg, bias=bias)
    return d
