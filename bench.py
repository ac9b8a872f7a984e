#!/usr/bin/env python
"""Benchmark: microseconds per routed MXFP4 MoE layer call on B200.

Headline workload: the largest single-GPU configuration, the DeepSeek-V3-class routed layer
(H=7168, I=2048, E=256, top-8, ~6 GB of MXFP4 weights) at M=512 tokens, where nearly every expert
is hit and the tensor-core path runs.  Before it, one line per other workload (the tiny layer, the
decode-width layer at M=1..8, the DeepSeek-class layer at M=1..32 and 256, the skewed layer at
M=1024) from the same run; the driver reads the last line.  Synthetic seeded inputs (moe_inputs),
weights resident in HBM, L2 flushed before every timed call by reading a 512 MB buffer (a read
leaves no dirty lines for the layer's kernels to write back).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config C] [--M M] [--sweep] [--headline-only]

Legs of the headline (one JSON line on rank 0):
  * timed: K CUDA-graph replays of one moe_mxfp4_forward_ex call, each bracketed
    by CUDA events on the replay stream; value = mean us/call (max over ranks);
  * kernel roofline: per-launch event times from moe_mxfp4_forward_profile; the
    dominant launch's algorithmic bytes (or FLOPs, when the call is tensor-bound) / time
    against the measured peak;
  * e2e: the same call through the C ABI from pinned HOST buffers, the x upload and
    the out download inside the timed region;
  * cpu_baseline: the fp64 oracle on the host cores (rank 0, N=1), on a bounded
    sample of the same workload.
`--impl reference` is the reference arm: the fp64 oracle alone, full layer calls on the host cores.
With N>1 (torchrun) the layer is split over the N GPUs along the expert intermediate dimension
(decode_moe_layer_b200.sharded): each rank streams I/N of every expert, the ranks all-gather their
fp32 [M,H] shares over NCCL and each reduces them in rank order; one step = the whole split call,
timed eagerly (the collective sits inside it), max over ranks, strong scaling.
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
CSRC = os.path.join(ROOT, "decode_moe_layer_b200", "csrc")
# committed ncu summaries that give a launch's DRAM bytes for a workload, with the hash of the
# kernel source they were taken on: (workload name, launch) -> (kernel source, summary)
TRAFFIC_PROFILES = {
    ("dsv3_wide_h7168_i2048_e256_k8 M=512", "gate_up_tc_small"):
        ([os.path.join(CSRC, f) for f in ("grouped_wide.cu", "common.cuh", "tcgen05.cuh", "moe_internal.h")],
         os.path.join(ROOT, "profiles", "grouped_wide_dsv3_h7168_i2048_e256_k8_M512.md")),
    ("dsv3_h7168_i2048_e256_k8 M=32", "gate_up"):
        ([os.path.join(CSRC, f) for f in ("grouped_gemm.cu", "common.cuh", "moe_internal.h")],
         os.path.join(ROOT, "profiles", "grouped_mxfp4_dsv3_h7168_i2048_e256_k8_M32.md")),
    ("decode_h2048_i768_e128_k8 M=8", "gate_up"):
        ([os.path.join(CSRC, f) for f in ("grouped_gemm.cu", "common.cuh", "moe_internal.h")],
         os.path.join(ROOT, "profiles", "grouped_mxfp4_decode_h2048_i768_e128_k8_M8.md")),
}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--config", type=int, default=3)
    p.add_argument("--M", type=int, default=512)
    p.add_argument("--sweep", action="store_true", help="one line per (config, M) of the workloads, no baselines")
    p.add_argument("--headline-only", action="store_true", help="skip the other workloads' lines")
    p.add_argument("--other-steps", type=int, default=20, help="timed steps of the non-headline lines")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--shape", default=None, metavar="H,I,E,k",
                   help="time one layer of this shape at --M instead of the workloads (same input recipe as "
                        "the tiny workload; e.g. a reduced expert count for a profiler capture)")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------- algorithmic work

# The library's split of an expert's assignments (moe_internal.h): tensor-core tiles when H and I are
# multiples of 512, M >= 5 and the experts average >= 2.5 assignments, for the experts with 5 or
# more (small tiles up to 64, large tiles above); mma.sync tiles for the others.
WIDE_MIN_TOKENS, WIDE_SMALL_MAX = 5, 64


def wide_on(shape, M):
    return (M >= WIDE_MIN_TOKENS and shape.H % 512 == 0 and shape.I % 512 == 0
            and 2 * M * shape.k >= WIDE_MIN_TOKENS * shape.E)


def down_fused(shape, M):
    """The library runs down and the weighted combine as one launch at the smallest sizes: M <= 8,
    I <= 1024, tiles of 8 assignments (M*k < 6E), no tensor-core tiles and at most 8 tiles."""
    return (1 <= M <= 8 and shape.I <= 1024 and M * shape.k < 6 * shape.E and not wide_on(shape, M)
            and min(M * shape.k, shape.E) <= 8)


def expert_classes(shape, M, ids):
    """Per-expert assignment counts and class ('narrow', 'small', 'large') from the realised routing."""
    H, I, E, k = shape.H, shape.I, shape.E, shape.k
    counts = np.bincount(np.asarray(ids).reshape(-1), minlength=E)
    wide = wide_on(shape, M)
    cls = {}
    for e in range(E):
        c = int(counts[e])
        if c == 0:
            continue
        if wide and c >= WIDE_MIN_TOKENS:
            cls[e] = "small" if c <= WIDE_SMALL_MAX else "large"
        else:
            cls[e] = "narrow"
    return counts, cls


def algorithmic(shape, M, ids):
    """Bytes and FLOPs the method must move/do for one call, from the realised routing, in total
    and per launch (the launches of moe_mxfp4_forward_profile)."""
    H, I, E, k = shape.H, shape.I, shape.E, shape.k
    counts, cls = expert_classes(shape, M, ids)
    touched = len(cls)
    w_bytes = touched * (51 * I * H // 32)
    total = w_bytes + E * H * 4 + 2 * M * H * 2 + M * k * 8
    flops = 6 * I * H * M * k + 2 * M * E * H
    per = {"route_logits": {"bytes": E * H * 4 + M * H * 2, "flops": 2 * M * E * H}}
    for name, kind in (("gate_up", "narrow"), ("gate_up_tc_small", "small"), ("gate_up_tc_large", "large"),
                       ("down", "narrow"), ("down_tc_small", "small"), ("down_tc_large", "large")):
        ex = [e for e, c in cls.items() if c == kind]
        n_assign = int(sum(counts[e] for e in ex))
        if name.startswith("gate_up"):
            b = len(ex) * (2 * I * H * 17 // 32) + n_assign * H * 2 + n_assign * I * 2
            f = 4 * I * H * n_assign
        elif name == "down" and down_fused(shape, M):   # with the combine: bf16 out, no fp32 rows
            b = len(ex) * (I * H * 17 // 32) + n_assign * I * 2 + M * k * 4 + M * H * 2
            f = 2 * I * H * n_assign
        else:
            b = len(ex) * (I * H * 17 // 32) + n_assign * I * 2 + n_assign * H * 4
            f = 2 * I * H * n_assign
        per[name] = {"bytes": b, "flops": f, "experts": len(ex), "assignments": n_assign}
    per["combine"] = {"bytes": M * k * H * 4 + M * k * 4 + M * H * 2, "flops": 0}
    return {"touched": touched, "bytes": total, "flops": flops, "weight_bytes": w_bytes, "per_launch": per,
            "classes": {kind: sum(1 for c in cls.values() if c == kind) for kind in ("narrow", "small", "large")}}


def kernel_code_hash(paths):
    """sha256[:16] of a kernel's sources (its file and the headers it includes, in order) with
    comments and blank space removed: any change to their code changes it, a change to their
    comments or layout does not."""
    code = []
    for path in paths:
        with open(path) as f:
            src = f.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        code.append(" ".join(src.split()))
    return hashlib.sha256("\n".join(code).encode()).hexdigest()[:16]


def profiled_traffic(workload, launch):
    """DRAM bytes of one launch from the committed ncu summary, if the kernel is unchanged since."""
    src, path = TRAFFIC_PROFILES.get((workload, launch), (None, None))
    if path is None or not os.path.exists(path):
        return None
    text = open(path).read()
    h = re.search(r"kernel code sha256\[:16\]:\s*([0-9a-f]+)", text)
    t = re.search(r"dram bytes per launch:\s*([0-9.eE+]+)", text)
    if not h or not t or h.group(1) != kernel_code_hash(src):
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
    tabs = [{}, {}, {}, {}]
    times = []
    t_start = time.perf_counter()
    step = 0
    while step < max_steps:
        elapsed = time.perf_counter() - t_start
        if step >= 2 and (elapsed >= min_seconds or elapsed >= max_seconds):
            break
        toks = tokens_per_step[step % len(tokens_per_step)]
        # the experts this step's tokens use, regenerated on the host (outside the step's timer)
        for e in sorted(set(int(e) for t in toks for e in ids[t])):
            if e not in tabs[0]:
                for i, v in enumerate(inp.expert_weights(e)):
                    tabs[i][e] = v
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
    # each step: the oracle on one group of tokens (the whole call when M is small; else enough tokens
    # to keep every host core busy, the time scaled by M / tokens), so that a step of the largest
    # workload takes seconds, not minutes.  The timed steps stop once REF_MAX_SECONDS have passed.
    subsets, n_tok = oracle_token_sample(M, shape.k)
    warm = time_oracle(inp, subsets, float("inf"), args.warmup, REF_MAX_WARMUP_SECONDS)[0] if args.warmup > 0 else []
    times, cores = time_oracle(inp, subsets, float("inf"), args.steps, REF_MAX_SECONDS)
    us_call = statistics.mean(times) * 1e6 * M / n_tok
    rec = {
        "impl": "reference", "metric": METRIC, "value": us_call, "unit": UNIT, "n_gpus": args.gpus,
        "steps": len(times), "warmup": len(warm), "ms_per_step": us_call / 1e3,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(workload_config(shape, M), timing="fp64 oracle on the host cores, wall clock"),
        "cpu_baseline": {"value": us_call, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": oracle_sample_text(len(times), n_tok, M) +
                         ", after %d untimed ones (%d and %d requested; timed steps stop after %d s, warm-up after "
                         "%d s)" % (len(warm), args.steps, args.warmup, REF_MAX_SECONDS, REF_MAX_WARMUP_SECONDS)},
        "e2e": {"value": us_call, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(rec))
    return 0


def workload_config(shape, M):
    return {"workload": "%s M=%d" % (shape.name, M), "M": M, "H": shape.H, "I": shape.I, "E": shape.E,
            "top_k": shape.k, "weights": "MXFP4 (E2M1 + E8M0 per 32)", "l2": "flushed (512 MB read) before each call",
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

    every = [(ci, M) for ci, s in enumerate(gen.CONFIGS) for M in s.Ms]
    headline = (args.config, args.M)
    if args.sweep:
        cases = [(c, False) for c in every]
    elif args.headline_only:
        cases = [(headline, True)]
    else:   # the other workloads first (fewer steps, no baselines), the headline last
        cases = [(c, False) for c in every if c != headline] + [(headline, True)]

    if args.shape:
        H, I, E, k = (int(v) for v in args.shape.split(","))
        custom = gen.LayerShape("custom_h%d_i%d_e%d_k%d" % (H, I, E, k), H, I, E, k, (args.M,))
        cases = [((0, args.M), True)]
    for (ci, M), is_headline in cases:
        shape = custom if args.shape else gen.CONFIGS[ci]
        steps = args.steps if (is_headline or args.sweep) else min(args.steps, args.other_steps)
        if world > 1:
            rec = run_case_sharded(torch, moe, dist, barrier, world, rank, dev, shape, ci, M, args, peaks,
                                   peak_kind, steps=steps)
        else:
            rec = run_case(torch, moe, dist, barrier, world, rank, dev, shape, ci, M, args, peaks, peak_kind,
                           baselines=is_headline, steps=steps)
        if rank == 0:
            print(json.dumps(rec), flush=True)
        torch.cuda.empty_cache()
    if world > 1:
        dist.destroy_process_group()
    return 0


def max_over_ranks(dist, values, device):
    """Element-wise maximum of every rank's values; all ranks get it (a step's time is its slowest rank's)."""
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def run_case(torch, moe, dist, barrier, world, rank, dev, shape, ci, M, args, peaks, peak_kind, baselines, steps):
    H, I, E, k = shape.H, shape.I, shape.E, shape.k
    inp = gen.make_inputs(ci, M, shape=shape, weights="torch", device=dev)
    xb = torch.from_numpy(np.ascontiguousarray(inp.x).view(np.int16)).to(dev).view(torch.bfloat16)
    wr = torch.from_numpy(inp.router_w).to(dev)
    bias = None if inp.router_bias is None else torch.from_numpy(inp.router_bias).to(dev)
    w13q, w13s, w2q, w2s = inp.w13_q, inp.w13_s, inp.w2_q, inp.w2_s
    ws = torch.empty(moe.moe_workspace_bytes(M, H, I, E, k), dtype=torch.uint8, device=dev)
    out = torch.empty((M, H), dtype=torch.bfloat16, device=dev)
    ids = torch.empty((M, k), dtype=torch.int32, device=dev)
    flush = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)

    def flush_l2():
        # reads 512 MB (four L2 capacities): the layer's weights and activations leave L2, and the
        # lines the read brings in are clean, so no kernel of the call pays a write-back for them
        torch.sum(flush)

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
            flush_l2()
            graph.replay()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        barrier()
        for i in range(steps):
            flush_l2()
            ev[i][0].record(stream)
            graph.replay()
            ev[i][1].record(stream)
        barrier()
        step_ms = [a.elapsed_time(b) for a, b in ev]
    clk = clocks.stop()

    # ------------------------------------------------------------------ per-kernel attribution
    prof = {n: [] for n in moe.PROFILE_KERNELS}
    with torch.cuda.stream(stream):
        for i in range(max(10, min(steps, 50))):
            flush_l2()
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
        for i in range(args.warmup + steps):
            flush_l2()
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
    call_bound = "hbm" if work["bytes"] / hbm > work["flops"] / (tflops * 1e3) else "tensor"
    # the dominant launch and its own algorithmic work (route_select / permute / gather have none
    # in this accounting; they are never dominant at these sizes)
    dominant = max(kern_us, key=kern_us.get)
    dom = work["per_launch"].get(dominant, {"bytes": work["bytes"], "flops": work["flops"]})
    if call_bound == "hbm":
        roof = {"bound": "hbm", "achieved": dom["bytes"] / (kern_us[dominant] * 1e3), "peak": hbm, "unit": "GB/s",
                "algorithmic_bytes_per_launch": dom["bytes"]}
    else:   # the contraction binds: FLOPs against the sustained bf16 tensor peak
        roof = {"bound": "tensor", "achieved": dom["flops"] / (kern_us[dominant] * 1e6), "peak": tflops,
                "unit": "TFLOP/s", "algorithmic_flops_per_launch": dom["flops"]}
    roof["frac"] = roof["achieved"] / roof["peak"]
    traffic = profiled_traffic(workload_config(shape, M)["workload"], dominant)
    sorted_ms = sorted(step_ms)
    rec = {
        "metric": METRIC, "value": mean_us, "unit": UNIT, "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": mean_us / 1e3, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 (MXFP4 weights decoded exactly to bf16), fp32 accumulate", "data": "synthetic",
        "config": dict(workload_config(shape, M), parallelism="replicas" if world > 1 else "1 GPU"),
        "p10_us": sorted_ms[len(sorted_ms) // 10] * 1e3, "p50_us": statistics.median(step_ms) * 1e3,
        "p90_us": sorted_ms[(9 * len(sorted_ms)) // 10] * 1e3,
        "gbs": work["bytes"] / (mean_us * 1e3),
        "roofline_call": {"bound": call_bound,
                          "roofline_us": roof_us, "frac": roof_us / mean_us, "peaks": peak_kind,
                          "roofline_us_nominal": roof_nominal_us, "frac_nominal": roof_nominal_us / mean_us,
                          "algorithmic_bytes": work["bytes"], "flops": work["flops"],
                          "touched_experts": work["touched"]},
        "kernels_us": {n: v for n, v in kern_us.items() if v > 0},
        "expert_tiles": work["classes"],
        "roofline": dict(kernel=dominant, traffic=traffic, peak_kind=peak_kind, **roof),
        "e2e": {"value": e2e_us, "unit": UNIT, "h2d_bytes_per_step": M * H * 2, "d2h_bytes_per_step": M * H * 2,
                "path": "pinned host x -> moe_mxfp4_forward_ex (eager C-ABI call) -> pinned host out"},
        "gpu_launches": moe.moe_forward_launches(M, H, I, E, k) * steps,
        "clocks": clk,
    }
    if baselines and rank == 0 and world == 1 and not args.no_cpu_baseline:
        host = gen.make_inputs(ci, M, shape=shape, weights="none")
        subsets, n_tok = oracle_token_sample(M, k)
        times, cores = time_oracle(host, subsets, 10.0, 30, 30.0)
        rec["cpu_baseline"] = {"value": statistics.mean(times) * 1e6 * M / n_tok, "unit": UNIT, "cores": cores,
                               "kind": "oracle", "sample": oracle_sample_text(len(times), n_tok, M)}
    return rec


def run_case_sharded(torch, moe, dist, barrier, world, rank, dev, shape, ci, M, args, peaks, peak_kind, steps):
    """One workload on N GPUs, I-sharded: every rank holds its I/N slice of every expert, and a step
    is this rank's share, the all-gather of the shares and the fixed-order reduction."""
    from decode_moe_layer_b200 import sharded
    H, I, E, k = shape.H, shape.I, shape.E, shape.k
    inp = gen.make_inputs(ci, M, shape=shape, weights="torch", device=dev)
    layer = sharded.IShardedLayer(inp.w13_q, inp.w13_s, inp.w2_q, inp.w2_s, k, device=dev)
    inp.w13_q = inp.w13_s = inp.w2_q = inp.w2_s = None
    torch.cuda.empty_cache()
    Is = layer.I_shard
    part_shape = gen.LayerShape(shape.name, H, Is, E, k, shape.Ms, shape.skew_bias)
    xb = torch.from_numpy(np.ascontiguousarray(inp.x).view(np.int16)).to(dev).view(torch.bfloat16)
    wr = torch.from_numpy(inp.router_w).to(dev)
    bias = None if inp.router_bias is None else torch.from_numpy(inp.router_bias).to(dev)
    out = torch.empty((M, H), dtype=torch.bfloat16, device=dev)
    ids = torch.empty((M, k), dtype=torch.int32, device=dev)
    flush = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)

    def step(x=xb, o=out):
        return layer.forward(x, wr, router_bias=bias, out=o)

    layer.partial(xb, wr, router_bias=bias, topk_ids_out=ids)
    torch.cuda.synchronize()
    work = algorithmic(part_shape, M, ids.cpu().numpy())
    clocks = ClockSampler(dev.index)
    for _ in range(args.warmup):
        torch.sum(flush)
        step()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier()
    for i in range(steps):
        torch.sum(flush)
        ev[i][0].record()
        step()
        ev[i][1].record()
    barrier()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    clk = clocks.stop()

    # per-kernel attribution of this rank's share (the same kernels; the profile form rounds out)
    ws = layer.workspace(M)
    prof = {n: [] for n in moe.PROFILE_KERNELS}
    for _ in range(10):
        torch.sum(flush)
        torch.cuda._sleep(2_000_000)
        _, ms = moe.moe_mxfp4_forward_profile(xb, wr, layer.w13_q, layer.w13_s, layer.w2_q, layer.w2_s, k, ws,
                                              router_bias=bias)
        for n, v in ms.items():
            prof[n].append(v)
    kern_us = {n: statistics.mean(v) * 1e3 for n, v in prof.items()}

    x_host = torch.empty((M, H), dtype=torch.bfloat16, pin_memory=True)
    x_host.copy_(xb.cpu())
    out_host = torch.empty((M, H), dtype=torch.bfloat16, pin_memory=True)
    x_dev = torch.empty_like(xb)
    e2e_ms = []
    for i in range(args.warmup + steps):
        torch.sum(flush)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        x_dev.copy_(x_host, non_blocking=True)
        step(x=x_dev)
        out_host.copy_(out, non_blocking=True)
        b.record()
        b.synchronize()
        if i >= args.warmup:
            e2e_ms.append(a.elapsed_time(b))
    barrier()
    mean_us, e2e_us = max_over_ranks(dist, [statistics.mean(step_ms) * 1e3, statistics.mean(e2e_ms) * 1e3], dev)

    hbm = peaks["hbm_gbs"]
    tflops = peaks["bf16_tflops_sustained"]
    # every rank streams its own slice at the same time: one rank's work sets the roofline
    roof_us = max(work["bytes"] / (hbm * 1e3), work["flops"] / (tflops * 1e6))
    call_bound = "hbm" if work["bytes"] / hbm > work["flops"] / (tflops * 1e3) else "tensor"
    dominant = max(kern_us, key=kern_us.get)
    dom = work["per_launch"].get(dominant, {"bytes": work["bytes"], "flops": work["flops"]})
    if call_bound == "hbm":
        roof = {"bound": "hbm", "achieved": dom["bytes"] / (kern_us[dominant] * 1e3), "peak": hbm, "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": dom["flops"] / (kern_us[dominant] * 1e6), "peak": tflops,
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    exchange = M * H * 4 * (world - 1)
    return {
        "metric": METRIC, "value": mean_us, "unit": UNIT, "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": mean_us / 1e3, "higher_is_better": False, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16 (MXFP4 weights decoded exactly to bf16), fp32 accumulate",
        "data": "synthetic",
        "config": dict(workload_config(shape, M), parallelism="I-shard %d (I/%d = %d per GPU)" % (world, world, Is),
                       timing="eager steps (this rank's share, NCCL all-gather, fixed-order reduction), CUDA "
                              "events on the current stream, max over ranks"),
        "roofline_call": {"bound": call_bound, "roofline_us": roof_us, "frac": roof_us / mean_us,
                          "peaks": peak_kind, "algorithmic_bytes_per_gpu": work["bytes"],
                          "exchange_bytes_per_gpu": exchange, "touched_experts": work["touched"]},
        "kernels_us": {n: v for n, v in kern_us.items() if v > 0},
        "roofline": dict(kernel=dominant, traffic=None, peak_kind=peak_kind, **roof),
        "e2e": {"value": e2e_us, "unit": UNIT, "h2d_bytes_per_step": M * H * 2, "d2h_bytes_per_step": M * H * 2,
                "path": "pinned host x -> IShardedLayer.forward (share, NCCL all-gather, reduce) -> pinned host out"},
        "gpu_launches": (moe.moe_forward_launches(M, H, Is, E, k) + 1) * steps,
        "clocks": clk,
    }


def oracle_token_sample(M, k, cores=None):
    """Token subsets for timing the oracle: the whole call when M is small, else disjoint groups of
    enough tokens (4 assignments per host core) to keep every core busy, each step's time scaled by
    M / tokens per step."""
    import oracle
    cores = cores or oracle.num_threads()
    n = min(M, max(1, -(-4 * cores // k)))
    groups = [list(range(i, min(M, i + n))) for i in range(0, M, n)]
    groups = [g for g in groups if len(g) == n] or [list(range(M))]
    return groups, n


def oracle_sample_text(steps, n_tok, M):
    if n_tok >= M:
        return "%d full layer calls (all %d tokens) of the same workload" % (steps, M)
    return ("%d oracle calls on disjoint groups of %d of the workload's %d tokens (all their %d assignments "
            "and the full routing), each scaled by %d/%d to one call" % (steps, n_tok, M, n_tok * 8, M, n_tok))


if __name__ == "__main__":
    sys.exit(main())
