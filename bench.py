"""Benchmark of the B200 routed-expert FFN layer (DeepSeek-V4.1-Flash shape).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one whole layer invocation (router, top-k, permutation, gate/up and
down grouped GEMMs, combine) on one batch of T synthetic tokens with the
weights resident in HBM. Prints one JSON line on rank 0.

  value      tokens/s over all ranks, timed with CUDA events around K steps
             (barrier + synchronize on both sides, max over ranks)
  e2e        the same metric through moe_forward_host_async (pinned host x in,
             y out): every step's x copied host->device and its y copied back
             inside the timed region, on the library's copy streams, overlapping
             the neighbouring steps' layers
  roofline   the dominant kernel's algorithmic bytes per launch / its mean
             launch time (CUDA events recorded by the library on the launch
             stream during the timed steps) against the measured HBM peak
  cpu_baseline  the float64 CPU oracle on a bounded sample of the same
             workload on this host's cores

Multi-GPU: the layer does not shard across GPUs in this build ("replicas
only"): every rank runs its own replica on its own tokens; no collective is on
the data path (one all-reduce of the elapsed time, for the max over ranks).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from routed_expert_ffn_sqrtsoftplus_b200 import synth  # noqa: E402

L2_BYTES = 126 * 1024 * 1024


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--workload", default="flash_decode", choices=sorted(synth.WORKLOADS))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--tokens", type=int, default=None, help="override T of the workload")
    p.add_argument("--experts", type=int, default=None,
                   help="override the routed expert count (small instances for profiler captures)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-secondary", action="store_true",
                   help="only the headline workload (skip the MXFP4 and prefill lines)")
    p.add_argument("--no-read-peak", action="store_true",
                   help="skip the read-only streaming peak (its 4 GiB buffer), e.g. under a profiler")
    p.add_argument("--cpu-seconds", type=float, default=15.0, help="budget of the CPU baseline sample")
    return p.parse_args()


# ----------------------------------------------------------------------------- distributed
def dist_setup(args):
    """One process per GPU (torchrun env); NCCL with GPUs, gloo on a host without
    them (only the oracle reference arm runs there). The process group's timeout is
    short so ranks that wait on a lost peer end with an error."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    gpu = torch.cuda.is_available()
    if world > 1:
        import datetime
        import torch.distributed as dist
        if gpu:
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    elif gpu:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    """The largest of the ranks' values (device times are reported as the max over ranks)."""
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(world: int, tokens_per_rank: int, steps: int, ms_max: float) -> float:
    """Whole-job tokens/s: every rank runs `steps` layer calls of `tokens_per_rank`
    tokens; the job takes the slowest rank's time."""
    return world * tokens_per_rank * steps / (ms_max / 1e3)


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self.index = period_s, index
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------------------- workload
def workload_from_args(args):
    import dataclasses
    wl = synth.WORKLOADS[args.workload]
    if args.tokens:
        wl = wl.with_tokens(args.tokens)
    if args.experts:
        wl = dataclasses.replace(wl, E=args.experts, name=f"{wl.name}_e{args.experts}")
    return wl


def build_layer(wl, device):
    d = synth.make_layer(wl, device=device)
    mxq = None
    if wl.expert_dtype in ("mxfp4", "mxfp8"):
        from routed_expert_ffn_sqrtsoftplus_b200 import quantize_mxfp4, quantize_mxfp8
        quant = quantize_mxfp4 if wl.expert_dtype == "mxfp4" else quantize_mxfp8
        mxq = {}
        for n, s in (("w1", "s1"), ("w3", "s3"), ("w2", "s2")):
            mxq[n], mxq[s] = quant(d[n])
    return d, mxq


def algorithmic(wl, idx: np.ndarray, T: int):
    """Bytes and FLOPs one step must move / do (weights read once, x in, y out), for the
    whole step and for each GEMM kernel (its weights read once, its activation rows in
    and out once)."""
    H, I, E, S, k = wl.H, wl.I, wl.E, wl.n_shared, wl.k
    U = len(np.unique(idx))
    mx = wl.expert_dtype in ("mxfp4", "mxfp8")
    if mx:
        div = 2 if wl.expert_dtype == "mxfp4" else 1     # values per weight byte
        routed13 = (2 * I * H) // div + (2 * I * H) // 32
        routed2 = (H * I) // div + (H * I) // 32
        act = 1                                  # MXFP8 activation bytes per value
    else:
        routed13, routed2, act = 2 * I * H * 2, H * I * 2, 2
    shared13, shared2 = 2 * I * H * 2, H * I * 2
    rr, rs = T * k, S * T                        # routed and shared rows
    step_bytes = U * (routed13 + routed2) + S * (shared13 + shared2) + E * H * 2 + 2 * T * H * 2
    step_flops = 2 * T * E * H + (rr + rs) * 3 * 2 * H * I
    kern = {}
    if mx:
        kern["gemm_gateup_mx"] = (U * routed13 + rr * (H + I) * act, rr * 4 * H * I)
        kern["gemm_down_mx"] = (U * routed2 + rr * I * act + rr * H * 4, rr * 2 * H * I)
        kern["gemm_gateup"] = (S * shared13 + rs * (H + I) * 2, rs * 4 * H * I)
        kern["gemm_down"] = (S * shared2 + rs * I * 2 + rs * H * 4, rs * 2 * H * I)
    else:
        kern["gemm_gateup"] = (U * routed13 + S * shared13 + (rr + rs) * (H + I) * 2, (rr + rs) * 4 * H * I)
        kern["gemm_down"] = (U * routed2 + S * shared2 + (rr + rs) * (I * 2 + H * 4), (rr + rs) * 2 * H * I)
        # few tokens: gate/up and down run as one launch
        kern["gemm_fused"] = (kern["gemm_gateup"][0] + kern["gemm_down"][0],
                              kern["gemm_gateup"][1] + kern["gemm_down"][1])
    return dict(U=U, step_bytes=step_bytes, step_flops=step_flops, kern=kern, rows=rr + rs)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def source_digest(files) -> str:
    """First 16 hex digits of the SHA-256 over the named csrc files, in order."""
    h = hashlib.sha256()
    for name in files:
        with open(os.path.join(ROOT, "routed_expert_ffn_sqrtsoftplus_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if the kernel's sources are unchanged since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        ent = rec[workload][kernel]
        return ent["bytes_per_launch"] if source_digest(ent["sources"]) == ent["sources_sha256_16"] else None
    except Exception:
        return None


# ----------------------------------------------------------------------------- CPU oracle baseline
def cpu_oracle_sample(wl, d, mxq, tokens, budget_s):
    """Time the float64 oracle on `tokens` (one token at a time, streaming each
    expert's weights from the device and upcasting them, until budget_s)."""
    from oracle import moe as om
    from oracle import mx as omx

    def f64(t):
        return t.detach().cpu().to(torch.float64).numpy()

    wg = f64(d["wg"])
    bias = None if d.get("bias") is None else f64(d["bias"])
    if mxq is None:
        routed = lambda e: (f64(d["w1"][e]), f64(d["w3"][e]), f64(d["w2"][e]))
    else:
        dqf = omx.dequantize_mxfp8 if wl.expert_dtype == "mxfp8" else omx.dequantize_mxfp4_packed
        dq = lambda n, s, e: dqf(mxq[n][e].cpu().numpy(), mxq[s][e].cpu().numpy())
        routed = lambda e: (dq("w1", "s1", e), dq("w3", "s3", e), dq("w2", "s2", e))
    shared = lambda j: (f64(d["sh_w1"][j]), f64(d["sh_w3"][j]), f64(d["sh_w2"][j]))
    ex = om.ExpertSource(routed, shared, wl.E, wl.n_shared, routed_is_mx=mxq is not None)
    done = 0
    t0 = time.perf_counter()
    for t in tokens:
        x = f64(d["x"][t:t + 1])
        om.moe_forward(x, wg, ex, wl.k, wl.route_scale, wl.swiglu_limit, bias=bias)
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return done, dt


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count()


# ----------------------------------------------------------------------------- main arms
def read_stream_peak(dev, gib: float = 4.0, reps: int = 5):
    """Read-only streaming bandwidth of this GPU in GB/s (moe_read_bandwidth: one CTA
    per SM keeps six 32 KiB bulk copies in flight over a 4 GiB buffer, far larger
    than L2, and computes nothing). The GEMMs' weight streams only read, so this
    is the ceiling they can approach; the copy bandwidth of MEASURED_PEAKS.json
    counts a read and a write per byte."""
    import routed_expert_ffn_sqrtsoftplus_b200 as moe
    buf = torch.ones(int(gib * (1 << 30)) // 4, dtype=torch.int32, device=dev)
    try:
        return moe.read_bandwidth(buf, reps)
    finally:
        del buf
        torch.cuda.empty_cache()


def kernel_roofline(kern, prof, alg, hbm, tc, src, read_gbs, wl_name):
    """Roofline of one kernel: algorithmic bytes (or FLOPs) per launch over its mean
    launch time (CUDA events on the launch stream), against the measured peaks."""
    k_ms, k_launch = prof[kern]
    k_avg_s = k_ms / k_launch / 1e3
    a_bytes, a_flops = alg["kern"].get(kern, (alg["step_bytes"], alg["step_flops"]))
    # block-scaled MXF8 x MXF4/MXF8 MMAs run at the FP8 rate: twice the measured BF16 peak (nominal 4.5 / 2.25)
    tc_k = tc * 2 if kern.endswith("_mx") else tc
    t_hbm = a_bytes / (hbm * 1e9)
    t_tc = a_flops / (tc_k * 1e12)
    if t_hbm >= t_tc:
        roof = {"bound": "hbm", "achieved": a_bytes / k_avg_s / 1e9, "peak": hbm, "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": a_flops / k_avg_s / 1e12, "peak": tc_k, "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = recorded_traffic(wl_name, kern)
    roof["kernel"] = kern
    roof["peak_source"] = (f"{src} (MEASURED_PEAKS.json)" if src == "measured" else "fallback") + \
        (", MXF8 = 2 x BF16" if kern.endswith("_mx") and roof["bound"] == "tensor" else "")
    if roof["bound"] == "hbm" and read_gbs:
        roof["read_peak_gbs"] = read_gbs
        roof["frac_of_read_peak"] = roof["achieved"] / read_gbs
    roof["achieved_tflops"] = a_flops / k_avg_s / 1e12
    roof["launch_ms"] = k_avg_s * 1e3
    return roof


def measure(wl, steps, warmup, world, local, read_gbs=None, flush_l2=False, e2e_steps=None, keep_weights=False):
    """Create the layer for workload `wl`, time `steps` forwards (inputs resident),
    attribute device time per kernel, time the host-buffer path, free the layer.
    Returns (results, the generated inputs, the MXFP4 tensors or None); the expert
    weights are dropped from the inputs unless keep_weights. Every rank runs the
    same steps in the same order."""
    import routed_expert_ffn_sqrtsoftplus_b200 as moe
    T = wl.T
    dev = torch.device("cuda", local)
    d, mxq = build_layer(wl, dev)
    layer = moe.MoELayer.from_layer(d, top_k=wl.k, max_tokens=T, route_scale=wl.route_scale,
                                    swiglu_limit=wl.swiglu_limit, mx=mxq)
    if not keep_weights:
        mxq = None
        for n in ("w1", "w3", "w2", "sh_w1", "sh_w3", "sh_w2"):
            d.pop(n, None)               # the library holds its own copy
        torch.cuda.empty_cache()
    x = d["x"]
    y = torch.empty_like(x)
    stream = torch.cuda.current_stream()
    _, idx, _ = layer.forward_with_routing(x)
    torch.cuda.synchronize()
    alg = algorithmic(wl, idx.cpu().numpy(), T)
    for _ in range(warmup):
        layer.forward(x, out=y)
    torch.cuda.synchronize()
    if layer.status() != moe.MOE_OK:
        raise RuntimeError(f"device status after the warm-up of {wl.name}")

    # ---- device-timed region
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for _ in range(steps):
            layer.forward(x, out=y)
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    if layer.status() != moe.MOE_OK:
        raise RuntimeError(f"device status after the timed steps of {wl.name}")
    ms = max_over_ranks(ev0.elapsed_time(ev1), world)
    res = {"value": weak_scaling_value(world, T, steps, ms), "ms_per_step": ms / steps, "steps": steps,
           "warmup": warmup, "clocks": clk.summary()}

    # ---- L2 flushed: a buffer twice the L2 size written before every timed step
    if flush_l2:
        # every step's flush, events and forward enqueued back to back (the host never
        # waits in between, so no step waits for its launches); the step time is the
        # sum of the per-step event intervals, which exclude the flushes
        junk = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i in range(steps):
            junk.fill_(float(i))
            evs[i][0].record(stream)
            layer.forward(x, out=y)
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        tot = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), world)
        del junk
        res["l2_flushed"] = {"value": weak_scaling_value(world, T, steps, tot), "ms_per_step": tot / steps,
                             "flush": f"{2 * L2_BYTES >> 20} MiB written before each step, outside its events"}

    # ---- per-kernel attribution: the same steps again with the library's CUDA events
    # on the launch stream around every kernel (an event between two kernels also keeps
    # the second from starting early, so these times are a little longer)
    layer.profile_begin(steps)
    for _ in range(steps):
        layer.forward(x, out=y)
    torch.cuda.synchronize()
    prof = layer.profile_end()
    if layer.status() != moe.MOE_OK:
        raise RuntimeError(f"device status after the attribution pass of {wl.name}")

    # ---- end to end through host buffers (pinned x in, y out, inside the timed region):
    # the pipelined host path, each step's x copied in and y copied out on the library's
    # copy streams while the neighbouring steps' layers run; three rotating buffer pairs,
    # since a call's buffers stay in use until two later calls have been issued
    xh = [x.cpu().pin_memory() for _ in range(3)]
    yh = [torch.empty_like(xh[0]).pin_memory() for _ in range(3)]
    n_e2e = e2e_steps or max(3, min(steps, 50))
    for i in range(3):
        layer.forward_host_async(xh[i], yh[i])
    layer.forward_host_wait()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(n_e2e):
        layer.forward_host_async(xh[i % 3], yh[i % 3])
    layer.forward_host_wait()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    res["e2e"] = {"value": weak_scaling_value(world, T, n_e2e, e2e_ms), "unit": "tokens/s",
                  "h2d_bytes_per_step": T * wl.H * 2, "d2h_bytes_per_step": T * wl.H * 2}

    hbm, tc, tc_sus, src = peaks()
    kern = max(prof, key=lambda n: prof[n][0])          # the kernel with the largest share of device time
    res["roofline"] = kernel_roofline(kern, prof, alg, hbm, tc, src, read_gbs, wl.name)
    res["kernel_rooflines"] = {n: kernel_roofline(n, prof, alg, hbm, tc, src, read_gbs, wl.name)
                               for n in prof if n in alg["kern"] and n != kern}
    step_s = res["ms_per_step"] / 1e3
    res["layer_roofline"] = {"bytes": alg["step_bytes"], "flops": alg["step_flops"],
                             "hbm_frac": alg["step_bytes"] / step_s / (hbm * 1e9),
                             "tensor_frac": alg["step_flops"] / step_s / (tc * 1e12),
                             "distinct_experts": alg["U"]}
    if read_gbs:
        res["layer_roofline"]["read_peak_frac"] = alg["step_bytes"] / step_s / (read_gbs * 1e9)
    res["kernels_ms_per_step"] = {n: v[0] / steps for n, v in sorted(prof.items())}
    res["gpu_launches"] = sum(c for _, c in prof.values())
    res["config"] = {"workload": wl.name, "T": T, "hidden": wl.H, "inter": wl.I, "n_routed": wl.E,
                     "n_shared": wl.n_shared, "top_k": wl.k, "route_scale": wl.route_scale,
                     "swiglu_limit": wl.swiglu_limit, "expert_dtype": wl.expert_dtype,
                     "parallelism": f"replicas x{world}",
                     "l2": f"no flush: each step streams {alg['step_bytes'] / 1e9:.2f} GB of weights > 126 MB L2"}
    res["dtype"] = {"bf16": "bf16", "mxfp4": "mxfp4xmxfp8", "mxfp8": "mxfp8xmxfp8"}.get(wl.expert_dtype,
                                                                                      wl.expert_dtype)
    layer.close()
    return res, d, mxq


# Workloads measured after the headline inside the same run (one layer at a time),
# so the one JSON line covers the metric's BF16 and MXFP4 shapes.
SECONDARY = ("flash_mxfp4_decode", "flash_mxfp4_prefill", "flash_prefill", "flash_mxfp8_decode",
             "flash_mxfp8_prefill")


def run_ours(args, world, rank, local):
    from routed_expert_ffn_sqrtsoftplus_b200 import build
    if rank == 0:
        build.build()
    barrier(world)
    wl = workload_from_args(args)
    dev = torch.device("cuda", local)
    read_gbs = None if args.no_read_peak else read_stream_peak(dev)
    head, d, mxq = measure(wl, args.steps, args.warmup, world, local, read_gbs=read_gbs, flush_l2=True,
                           keep_weights=rank == 0 and world == 1 and not args.no_cpu_baseline)
    out = {
        "metric": "MoE layer tokens/s (Flash shape, BF16 & MXFP4) + % of HBM/tensor roofline",
        "value": head["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": head["dtype"],
        "data": "synthetic (seeded N(0,1/fan_in) BF16 weights, N(0,1) tokens)",
        "config": head["config"],
        "e2e": head["e2e"],
        "roofline": head["roofline"],
        "kernel_rooflines": head["kernel_rooflines"],
        "layer_roofline": head["layer_roofline"],
        "l2_flushed": head["l2_flushed"],
        "kernels_ms_per_step": head["kernels_ms_per_step"],
        "kernel_timing": "per-kernel CUDA events in a second pass of the same steps (roofline, kernels_ms_per_step)",
        "gpu_launches": head["gpu_launches"],
        "clocks": head["clocks"],
        "read_stream_peak_gbs": read_gbs,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rng = np.random.default_rng(0)
        toks = rng.permutation(wl.T)
        n, dt = cpu_oracle_sample(wl, d, mxq, toks, args.cpu_seconds)
        out["cpu_baseline"] = {"value": n / dt, "unit": "tokens/s", "cores": cpu_cores(), "kind": "oracle",
                               "sample": f"{n} of {wl.T} tokens, one at a time; each hit expert's weights copied "
                                         f"from the device and upcast to float64 inside the timing"}
    del d, mxq
    torch.cuda.empty_cache()
    if not args.no_secondary and args.workload == "flash_decode" and not args.tokens and not args.experts:
        sec = {}
        steps, warm = min(args.steps, 30), max(3, min(args.warmup, 5))
        for name in SECONDARY:
            r, dd, _ = measure(synth.WORKLOADS[name], steps, warm, world, local, read_gbs=read_gbs)
            del dd
            torch.cuda.empty_cache()
            sec[name] = {k: r[k] for k in ("value", "ms_per_step", "steps", "warmup", "dtype", "e2e", "roofline",
                                           "kernel_rooflines", "layer_roofline", "kernels_ms_per_step",
                                           "gpu_launches", "clocks", "config")}
            sec[name]["unit"] = "tokens/s"
        out["secondary"] = sec
    return out


def run_reference(args, world, rank, local):
    """The float64 CPU oracle as the reference arm, on rank 0 only."""
    wl = workload_from_args(args)
    if rank != 0:
        return None
    # inputs are drawn on the GPU like the other arm's; a host without one draws
    # them on the CPU (BF16 workloads only: the MXFP4 codec of the set-up runs on the GPU)
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    d, mxq = build_layer(wl, dev)
    # one token per step; the whole run stops at the time budget (an MXFP4 token
    # takes seconds on the host), having timed at least one step
    total_budget = 150.0
    per_step = max(0.2, total_budget / max(1, args.steps + args.warmup))
    rng = np.random.default_rng(1)
    done_t, dt_t, timed = 0, 0.0, 0
    t_start = time.perf_counter()
    for i in range(args.warmup + args.steps):
        if timed > 0 and time.perf_counter() - t_start > total_budget:
            break
        if i < args.warmup and time.perf_counter() - t_start > total_budget / 4:
            continue  # warm-up is cut short rather than the timed steps
        toks = rng.integers(0, wl.T, size=1)
        n, dt = cpu_oracle_sample(wl, d, mxq, toks, per_step)
        if i >= args.warmup:
            done_t += n
            dt_t += dt
            timed += 1
    value = done_t / dt_t
    return {
        "impl": "reference",
        "metric": "MoE layer tokens/s (Flash shape, BF16 & MXFP4) + % of HBM/tensor roofline",
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt_t / max(1, timed), "steps_sampled": timed, "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "T": wl.T, "hidden": wl.H, "inter": wl.I, "n_routed": wl.E,
                   "top_k": wl.k, "expert_dtype": wl.expert_dtype},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cpu_cores(), "kind": "oracle",
                         "sample": f"one token per step ({timed} timed steps within a {total_budget:.0f} s budget), "
                                   "its routed experts and the shared expert streamed from the device and "
                                   "upcast to float64"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    try:
        out = run_reference(args, world, rank, local) if args.impl == "reference" else run_ours(args, world, rank, local)
        if rank == 0 and out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
