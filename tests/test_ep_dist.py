"""Expert parallelism on CPU: the exchange plumbing of ExpertParallelLayer over a
gloo process group of two ranks, with the float64 oracle as each rank's partial
computation (the library's kernels need a GPU; their partial outputs are checked
against the oracle in tests/test_gpu_ep.py). No GPU is needed here.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from routed_expert_ffn_sqrtsoftplus_b200.ep import ExpertParallelLayer, expert_window  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer(T_total, seed=21):
    from routed_expert_ffn_sqrtsoftplus_b200 import synth
    wl = synth.Workload("ep_small", T=T_total, H=64, I=32, E=12, k=3, seed=seed)
    return wl, synth.make_layer(wl, device="cpu")


def _worker(rank, world, port, T_local, q):
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import parity
    from oracle import moe as om
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl, lay = _layer(T_local * world)
        b, c = expert_window(wl.E, world, rank)
        ex = parity.LayerExperts(lay)
        wg = parity.f64(lay["wg"])

        def partial(x_all):
            y = om.moe_forward_partial(parity.f64(x_all), wg, ex, wl.k, wl.route_scale, wl.swiglu_limit, b, b + c,
                                       include_shared=(rank == 0))
            return torch.from_numpy(y).to(torch.float32)

        ep = ExpertParallelLayer(partial)
        x_local = lay["x"][rank * T_local:(rank + 1) * T_local]
        y = ep(x_local)
        ref = om.moe_forward(parity.f64(x_local), wg, ex, wl.k, wl.route_scale, wl.swiglu_limit).y
        err = float(np.abs(y.double().numpy() - ref).max() / np.sqrt(np.mean(ref ** 2)))
        q.put((rank, b, c, err))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("T_local", [1, 5])
def test_expert_parallel_layer_over_two_gloo_ranks(T_local):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, world, port, T_local, q)) for r in range(world)]
    for p in ps:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in ps:
        p.join(60)
        assert p.exitcode == 0
    # the two windows partition the experts, and each rank's output is the layer's
    assert [(r[1], r[2]) for r in res] == [(0, 6), (6, 6)]
    for rank, b, c, err in res:
        assert err < 1e-6, f"rank {rank}: relative error {err}"


def test_expert_windows_partition_the_experts():
    for E in (1, 7, 12, 384, 512):
        for world in range(1, min(E, 9) + 1):
            wins = [expert_window(E, world, r) for r in range(world)]
            assert wins[0][0] == 0 and all(c >= 1 for _, c in wins)
            assert all(wins[i][0] + wins[i][1] == wins[i + 1][0] for i in range(world - 1))
            assert wins[-1][0] + wins[-1][1] == E
            assert max(c for _, c in wins) - min(c for _, c in wins) <= 1
    with pytest.raises(ValueError):
        expert_window(4, 5, 0)
