"""The multi-process side of bench.py on CPU: gloo process groups of two ranks.

Covers the max-over-ranks timing, the whole-job weak-scaling value and the
reference arm under torchrun (rank 0 alone prints the JSON line, every rank
exits 0). No GPU is needed.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        # rank r "took" 10 + r ms: the job time is the slowest rank's
        ms = bench.max_over_ranks(10.0 + rank, world)
        v = bench.weak_scaling_value(world, 32, 5, ms)
        q.put((rank, ms, v))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    mp.start_processes(_worker, args=(world, port, q), nprocs=world, join=True, start_method="spawn")
    got = sorted(q.get() for _ in range(world))
    for rank, ms, v in got:
        assert ms == 11.0
        assert v == pytest.approx(2 * 32 * 5 / 0.011)


def test_weak_scaling_value_single_rank():
    import bench
    assert bench.weak_scaling_value(1, 8192, 10, 62.0) == pytest.approx(8192 * 10 / 0.062)


@pytest.mark.timeout(600)
def test_reference_arm_under_torchrun_two_ranks():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           "bench.py", "--impl", "reference", "--workload", "tiny", "--gpus", "2", "--steps", "1", "--warmup", "1"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=540)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
