#!/usr/bin/env python
"""Benchmark: microseconds per routed MXFP4 MoE layer call on B200.

Default workload: the decode-width Qwen3-MoE-like layer (H=2048, I=768, E=128,
top-8) at M=8 tokens, the c8 decode point that "row/QUANT-CT-MXFP4-C8-DIFF"
(vllm.cpp PR #52) traces.  Synthetic seeded inputs (moe_inputs), weights resident
in HBM, L2 flushed (512 MB write) before every timed call.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config C] [--M M] [--sweep]

Legs of the default run (one JSON line on rank 0):
  * timed: K CUDA-graph replays of one moe_mxfp4_forward_ex call, each bracketed
    by CUDA events on the replay stream; value = mean us/call (max over ranks);
  * kernel roofline: per-kernel event times from moe_mxfp4_forward_profile; the
    dominant kernel's algorithmic bytes / time against the measured HBM peak;
  * e2e: the same call through the C ABI from pinned HOST buffers, the x upload and
    the out download inside the timed region;
  * cpu_baseline: the fp64 oracle on the host cores (rank 0, N=1), on a bounded
    sample of the same workload.
`--impl reference` is the reference arm: the fp64 oracle alone, full layer calls on the host cores.
With N>1 (torchrun) every rank runs an independent replica of the layer call.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from moe_inputs import generator as gen  # noqa: E402

METRIC = "routed MXFP4 MoE layer µs/call and HBM GB/s vs ~8 TB/s roofline, M=1–1024"
UNIT = "us/call"
NOMINAL_HBM_GBS = 8000.0
NOMINAL_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 512 << 20
KERNEL_SRC = os.path.join(ROOT, "decode_moe_layer_b200", "csrc", "grouped_gemm.cu")
TRAFFIC_PROFILE = os.path.join(ROOT, "profiles", "grouped_mxfp4_decode_h2048_i768_e128_k8_M8.md")


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--config", type=int, default=1)
    p.add_argument("--M", type=int, default=8)
    p.add_argument("--sweep", action="store_true", help="one line per (config, M) of the workloads, no baselines")
    p.add_argument("--no-cpu-baseline", action="store_true")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------- algorithmic work

def algorithmic(shape, M, ids):
    """Bytes and FLOPs the method must move/do for one call, from the realised routing."""
    H, I, E, k = shape.H, shape.I, shape.E, shape.k
    touched = len(np.unique(ids))
    w_bytes = touched * (51 * I * H // 32)
    total = w_bytes + E * H * 4 + 2 * M * H * 2 + M * k * 8
    flops = 6 * I * H * M * k + 2 * M * E * H
    gate_up = touched * (2 * I * H * 17 // 32) + M * H * 2 + M * k * I * 2
    down = touched * (I * H * 17 // 32) + M * k * I * 2 + M * H * 2
    return {"touched": touched, "bytes": total, "flops": flops, "weight_bytes": w_bytes,
            "gate_up_bytes": gate_up, "down_bytes": down,
            "gate_up_flops": 4 * I * H * M * k, "down_flops": 2 * I * H * M * k}


def kernel_code_hash(path=None):
    """sha256[:16] of the dominant kernel's source with comments and blank space removed: any change
    to its code changes it, a change to its comments or layout does not."""
    with open(path or KERNEL_SRC) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return hashlib.sha256(" ".join(src.split()).encode()).hexdigest()[:16]


def profiled_traffic():
    """dram bytes per launch of the dominant kernel from the committed ncu summary, if the kernel is unchanged."""
    if not os.path.exists(TRAFFIC_PROFILE):
        return None
    text = open(TRAFFIC_PROFILE).read()
    h = re.search(r"kernel code sha256\[:16\]:\s*([0-9a-f]+)", text)
    t = re.search(r"dram bytes per launch:\s*([0-9.eE+]+)", text)
    if not h or not t or h.group(1) != kernel_code_hash():
        return None
    return float(t.group(1))


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        import torch
        self.proc = None
        self.path = tempfile.mktemp(prefix="clocks_", suffix=".csv")
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            ident = ["-i", "GPU-" + uuid if not uuid.startswith("GPU-") else uuid]
        except Exception:
            ident = []
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                                          "-lms", "50"] + ident, stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
                power.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None, "samples": len(sm), "reasons": sorted(reasons)}


# --------------------------------------------------------------------------- CPU oracle

def time_oracle(inp, tokens_per_step, min_seconds, max_steps, max_seconds=float("inf")):
    """Seconds of each oracle call over the given token subsets (one subset per step): at least
    two steps, then more until min_seconds have passed, never more than max_steps, and no new
    step once max_seconds have passed."""
    import oracle
    shape = inp.shape
    ids, _, _ = oracle.route(inp.x, inp.router_w, inp.router_bias, shape.k)
    need = sorted(set(int(e) for e in ids.ravel()))
    ex = {e: inp.expert_weights(e) for e in need}
    tabs = [{e: v[i] for e, v in ex.items()} for i in range(4)]
    times = []
    t_start = time.perf_counter()
    step = 0
    while step < max_steps:
        elapsed = time.perf_counter() - t_start
        if step >= 2 and (elapsed >= min_seconds or elapsed >= max_seconds):
            break
        toks = tokens_per_step[step % len(tokens_per_step)]
        t0 = time.perf_counter()
        oracle.forward(inp.x, inp.router_w, inp.router_bias, tabs[0], tabs[1], tabs[2], tabs[3], shape.k,
                       tokens=toks, I=shape.I)
        times.append(time.perf_counter() - t0)
        step += 1
    return times, oracle.num_threads()


REF_MAX_SECONDS = 120
REF_MAX_WARMUP_SECONDS = 20


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    shape = gen.CONFIGS[args.config]
    M = args.M
    inp = gen.make_inputs(args.config, M, weights="none")
    # each step: one full layer call of the workload (all M tokens).  A one-token step scaled by M
    # would not do: the oracle spreads a call over its assignments and tokens, so one token leaves
    # most host cores idle.  The timed steps stop once REF_MAX_SECONDS have passed, so that a large
    # --steps still ends in minutes.
    full = [list(range(M))]
    warm = time_oracle(inp, full, float("inf"), args.warmup, REF_MAX_WARMUP_SECONDS)[0] if args.warmup > 0 else []
    times, cores = time_oracle(inp, full, float("inf"), args.steps, REF_MAX_SECONDS)
    us_call = statistics.mean(times) * 1e6
    rec = {
        "impl": "reference", "metric": METRIC, "value": us_call, "unit": UNIT, "n_gpus": args.gpus,
        "steps": len(times), "warmup": len(warm), "ms_per_step": statistics.mean(times) * 1e3,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(workload_config(shape, M), timing="fp64 oracle on the host cores, wall clock"),
        "cpu_baseline": {"value": us_call, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": "%d full layer calls (all %d tokens) of the same workload, one per step, "
                                   "after %d untimed ones (%d and %d requested; timed steps stop after %d s, "
                                   "warm-up after %d s)" % (len(times), M, len(warm), args.steps, args.warmup,
                                                            REF_MAX_SECONDS, REF_MAX_WARMUP_SECONDS)},
        "e2e": {"value": us_call, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(rec))
    return 0


def workload_config(shape, M):
    return {"workload": "%s M=%d" % (shape.name, M), "M": M, "H": shape.H, "I": shape.I, "E": shape.E,
            "top_k": shape.k, "weights": "MXFP4 (E2M1 + E8M0 per 32)", "l2": "flushed (512 MB write) before each call",
            "timing": "CUDA-graph replay of one moe_mxfp4_forward_ex call, CUDA events"}


# --------------------------------------------------------------------------- GPU legs

def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    import decode_moe_layer_b200 as moe
    sys.path.insert(0, os.path.join(ROOT, "tests"))

    peaks, peak_kind = load_peaks()

    cases = [(args.config, args.M)]
    if args.sweep:
        cases = [(ci, M) for ci, s in enumerate(gen.CONFIGS) for M in s.Ms]

    for ci, M in cases:
        shape = gen.CONFIGS[ci]
        rec = run_case(torch, moe, dist, barrier, world, rank, dev, shape, ci, M, args, peaks, peak_kind,
                       baselines=not args.sweep)
        if rank == 0:
            print(json.dumps(rec), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def max_over_ranks(dist, values, device):
    """Element-wise maximum of every rank's values; all ranks get it (a step's time is its slowest rank's)."""
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def run_case(torch, moe, dist, barrier, world, rank, dev, shape, ci, M, args, peaks, peak_kind, baselines):
    H, I, E, k = shape.H, shape.I, shape.E, shape.k
    inp = gen.make_inputs(ci, M, weights="torch", device=dev)
    xb = torch.from_numpy(np.ascontiguousarray(inp.x).view(np.int16)).to(dev).view(torch.bfloat16)
    wr = torch.from_numpy(inp.router_w).to(dev)
    bias = None if inp.router_bias is None else torch.from_numpy(inp.router_bias).to(dev)
    w13q, w13s, w2q, w2s = inp.w13_q, inp.w13_s, inp.w2_q, inp.w2_s
    ws = torch.empty(moe.moe_workspace_bytes(M, H, I, E, k), dtype=torch.uint8, device=dev)
    out = torch.empty((M, H), dtype=torch.bfloat16, device=dev)
    ids = torch.empty((M, k), dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()

    def call(o=out, x=xb, ids_out=None):
        return moe.moe_mxfp4_forward_ex(x, wr, w13q, w13s, w2q, w2s, k, ws, router_bias=bias, out=o,
                                        topk_ids_out=ids_out)

    with torch.cuda.stream(stream):
        call(ids_out=ids)
        stream.synchronize()
        work = algorithmic(shape, M, ids.cpu().numpy())
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            call()
    torch.cuda.synchronize()

    clocks = ClockSampler(dev.index)
    step_ms = []
    with torch.cuda.stream(stream):
        # soak: ~0.5 s of back-to-back replays so clocks settle and get sampled under load
        t_end = time.perf_counter() + 0.5
        while time.perf_counter() < t_end:
            for _ in range(50):
                graph.replay()
            stream.synchronize()
        for i in range(args.warmup):
            flush.fill_(i & 0xFF)
            graph.replay()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        barrier()
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            ev[i][0].record(stream)
            graph.replay()
            ev[i][1].record(stream)
        barrier()
        step_ms = [a.elapsed_time(b) for a, b in ev]
    clk = clocks.stop()

    # ------------------------------------------------------------------ per-kernel attribution
    prof = {n: [] for n in moe.PROFILE_KERNELS}
    with torch.cuda.stream(stream):
        for i in range(max(10, min(args.steps, 50))):
            flush.fill_(i & 0xFF)
            # a short device-side sleep queued first lets the host enqueue every kernel and
            # event of the call before the GPU reaches them: event gaps then hold device time only
            torch.cuda._sleep(2_000_000)
            _, ms = moe.moe_mxfp4_forward_profile(xb, wr, w13q, w13s, w2q, w2s, k, ws, router_bias=bias, out=out)
            for n, v in ms.items():
                prof[n].append(v)
    kern_us = {n: statistics.mean(v) * 1e3 for n, v in prof.items()}

    # ------------------------------------------------------------------ e2e from host buffers
    x_host = torch.empty((M, H), dtype=torch.bfloat16, pin_memory=True)
    x_host.copy_(xb.cpu())
    out_host = torch.empty((M, H), dtype=torch.bfloat16, pin_memory=True)
    x_dev = torch.empty_like(xb)
    e2e_ms = []
    with torch.cuda.stream(stream):
        for i in range(args.warmup + args.steps):
            flush.fill_(i & 0xFF)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            x_dev.copy_(x_host, non_blocking=True)
            call(x=x_dev)
            out_host.copy_(out, non_blocking=True)
            b.record(stream)
            b.synchronize()
            if i >= args.warmup:
                e2e_ms.append(a.elapsed_time(b))
    torch.cuda.synchronize()

    mean_us = statistics.mean(step_ms) * 1e3
    e2e_us = statistics.mean(e2e_ms) * 1e3
    if world > 1:
        mean_us, e2e_us = max_over_ranks(dist, [mean_us, e2e_us], dev)

    hbm = peaks["hbm_gbs"]
    tflops = peaks["bf16_tflops_sustained"]
    roof_us = max(work["bytes"] / (hbm * 1e3), work["flops"] / (tflops * 1e6))
    roof_nominal_us = max(work["bytes"] / (NOMINAL_HBM_GBS * 1e3), work["flops"] / (NOMINAL_BF16_TFLOPS * 1e6))
    dominant = max(kern_us, key=kern_us.get)
    dom_bytes = {"gate_up_swiglu": work["gate_up_bytes"], "down_combine": work["down_bytes"]}.get(dominant)
    if dom_bytes is None:
        dom_bytes = work["bytes"]
    dom_flops = {"gate_up_swiglu": work["gate_up_flops"], "down_combine": work["down_flops"]}.get(dominant,
                                                                                                   work["flops"])
    call_bound = "hbm" if work["bytes"] / hbm > work["flops"] / (tflops * 1e3) else "tensor"
    if call_bound == "hbm":
        roof = {"bound": "hbm", "achieved": dom_bytes / (kern_us[dominant] * 1e3), "peak": hbm, "unit": "GB/s",
                "algorithmic_bytes_per_launch": dom_bytes}
    else:   # the contraction binds: FLOPs against the sustained bf16 tensor peak
        roof = {"bound": "tensor", "achieved": dom_flops / (kern_us[dominant] * 1e6), "peak": tflops,
                "unit": "TFLOP/s", "algorithmic_flops_per_launch": dom_flops}
    roof["frac"] = roof["achieved"] / roof["peak"]
    traffic = profiled_traffic() if (ci, M) == (1, 8) and dominant == "gate_up_swiglu" else None
    sorted_ms = sorted(step_ms)
    rec = {
        "metric": METRIC, "value": mean_us, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": mean_us / 1e3, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "mxfp4 weights x f16 activations, fp32 accumulate", "data": "synthetic",
        "config": dict(workload_config(shape, M), parallelism="replicas" if world > 1 else "1 GPU"),
        "p10_us": sorted_ms[len(sorted_ms) // 10] * 1e3, "p50_us": statistics.median(step_ms) * 1e3,
        "p90_us": sorted_ms[(9 * len(sorted_ms)) // 10] * 1e3,
        "gbs": work["bytes"] / (mean_us * 1e3),
        "roofline_call": {"bound": call_bound,
                          "roofline_us": roof_us, "frac": roof_us / mean_us, "peaks": peak_kind,
                          "roofline_us_nominal": roof_nominal_us, "frac_nominal": roof_nominal_us / mean_us,
                          "algorithmic_bytes": work["bytes"], "flops": work["flops"],
                          "touched_experts": work["touched"]},
        "kernels_us": kern_us,
        "roofline": dict(kernel=dominant, traffic=traffic, peak_kind=peak_kind, **roof),
        "e2e": {"value": e2e_us, "unit": UNIT, "h2d_bytes_per_step": M * H * 2, "d2h_bytes_per_step": M * H * 2,
                "path": "pinned host x -> moe_mxfp4_forward_ex (eager C-ABI call) -> pinned host out"},
        "gpu_launches": moe.moe_forward_launches(M, H, I, E, k) * args.steps,
        "clocks": clk,
    }
    if baselines and rank == 0 and world == 1 and not args.no_cpu_baseline:
        host = gen.make_inputs(ci, M, weights="none")
        subsets = [list(range(M))]
        times, cores = time_oracle(host, subsets, 10.0, 30)
        rec["cpu_baseline"] = {"value": statistics.mean(times) * 1e6, "unit": UNIT, "cores": cores, "kind": "oracle",
                               "sample": "%d full layer calls (all %d tokens) of the same workload" % (len(times), M)}
    return rec


if __name__ == "__main__":
    sys.exit(main())
