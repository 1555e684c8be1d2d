"""The seeded workload generator: deterministic, right shapes and distributions."""
import math

import numpy as np
import torch

from routed_expert_ffn_sqrtsoftplus_b200 import synth


def test_workload_table_matches_pages():
    import json, os
    with open(os.path.join(os.path.dirname(__file__), "golden", "page_constants.json")) as f:
        pc = json.load(f)
    fl = synth.WORKLOADS["flash_decode"]
    assert (fl.H, fl.I, fl.E, fl.n_shared, fl.k) == (pc["dim"]["value"], pc["moe_inter_dim"]["value"],
                                                     pc["n_routed_experts"]["value"], pc["n_shared_experts"]["value"],
                                                     pc["n_activated_experts"]["value"])
    assert (fl.route_scale, fl.swiglu_limit) == (pc["route_scale"]["value"], pc["swiglu_limit"]["value"])
    pro = synth.WORKLOADS["pro_skewed"]
    assert (pro.H, pro.I) == (pc["pro_hidden"]["value"], pc["pro_moe_intermediate_size"]["value"])
    ds = synth.WORKLOADS["dspark"]
    assert (ds.E, ds.k) == (pc["dspark_n_routed_experts"]["value"], pc["dspark_n_activated_experts"]["value"])
    assert [synth.WORKLOADS[n].T for n in ("tiny", "flash_decode", "flash_prefill", "flash_mxfp4_decode",
                                           "flash_mxfp4_prefill", "pro_skewed")] == [64, 32, 8192, 16, 4096, 2048]


def test_deterministic_and_distributed():
    wl = synth.WORKLOADS["tiny"]
    a = synth.make_layer(wl)
    b = synth.make_layer(wl)
    for key in ("x", "wg", "w1", "w3", "w2", "sh_w1", "sh_w3", "sh_w2"):
        assert a[key].dtype == torch.bfloat16
        assert torch.equal(a[key], b[key]), key
    assert a["x"].shape == (64, 512) and a["w1"].shape == (32, 256, 512) and a["w2"].shape == (32, 512, 256)
    assert a["bias"] is None
    # variance 1/fan_in: router logits come out about N(0, 1)
    assert abs(a["x"].float().std().item() - 1.0) < 0.05
    assert abs(a["wg"].float().std().item() * math.sqrt(512) - 1.0) < 0.05
    assert abs(a["w2"].float().std().item() * math.sqrt(256) - 1.0) < 0.05
    z = a["x"].double() @ a["wg"].double().T
    assert 0.85 < z.std().item() < 1.15
    c = synth.make_layer(wl, seed=5)
    assert not torch.equal(a["w1"], c["w1"])


def test_zipf_bias():
    wl = synth.Workload("zipf_small", T=8, H=128, I=128, E=16, zipf_bias=True, seed=3)
    _, bias = synth.make_router(wl)
    ranks = np.exp(-bias.double().numpy() / 2.0)          # b = 2 ln(1/rank)  =>  rank = e^{-b/2}
    assert np.allclose(np.sort(ranks), np.arange(1, 17), rtol=1e-6)
    assert bias.max().item() == 0.0
