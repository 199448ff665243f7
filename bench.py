#!/usr/bin/env python3
"""Benchmark: matmul-only batch-1 decode of Qwen2.5-0.5B with Q8_0 weights.

One step = one decode token's matmul set, run through the libq8 C ABI:
24 layers x {qkv 1152x896 (GEMV), wo 896x896 (GEMV), gate_up 9728x896 with the
fused SiLU(gate)*up epilogue, down 896x4864 (GEMV)} + lm_head 151936x896
(GEMV): 97 launches, captured once in a CUDA graph and replayed.  Weights are
synthetic Q8_0 (q uniform in [-127, 127], d = |N(0,1)| * 0.02, one seed per
matrix), activations fp32 N(0,1), one fresh vector per matrix.  The 525 MB of
weights are larger than L2, so no flush is needed between steps.

Reports one JSON line (see --help): tokens/s over all GPUs, the HBM GB/s the
step achieves (34 bytes per 32 weights), the roofline of the dominant kernel,
an end-to-end figure with host copies, clocks seen during the timed region,
and the CPU oracle timed on the host as a baseline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {ours,reference}]

With N > 1 it runs under torchrun, one rank per GPU, each rank an independent
replica (the path has no exchange step); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import q8gen  # noqa: E402

METRIC = "Q8_0 GEMV achieved HBM GB/s (% of B200 peak); matmul-only decode tok/s at N=1"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
WORKLOAD = ("qwen2.5-0.5b batch-1 decode matmul set: 24 x {qkv 1152x896, wo 896x896, "
            "gate_up 9728x896 + SwiGLU, down 896x4864} + lm_head 151936x896, Q8_0 weights, fp32 x")


def max_over_ranks(value, world, device):
    """The largest `value` over the job's ranks, received by every rank: a
    job's time is its slowest rank's.  `value` itself with one rank."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(world, units_per_rank, elapsed_max):
    """Whole-job throughput of `world` independent replicas: the units all
    ranks processed over the slowest rank's time."""
    return world * units_per_rank / elapsed_max


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def algorithmic_bytes(M, K):
    return M * K * 34 // 32


# ---------------------------------------------------------------------------
# CPU oracle baseline
# ---------------------------------------------------------------------------

def oracle_decode_tokens(weights, xs, target_s=10.0, threads=None):
    """Time the fp64 CPU oracle on whole decode tokens until about target_s
    seconds of work are done.  Returns (tokens/s, tokens, seconds, threads)."""
    import oracle
    threads = threads or oracle.max_threads()
    tokens, t0 = 0, time.perf_counter()
    while True:
        for (spec, g), x in zip(weights, xs):
            if spec.swiglu:
                oracle.gate_up_swiglu(g, x, spec.M // 2, spec.K, threads=threads)
            else:
                oracle.gemv(g, x, spec.M, spec.K, threads=threads)
        tokens += 1
        dt = time.perf_counter() - t0
        if dt >= target_s:
            return tokens / dt, tokens, dt, threads


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [p.strip() for p in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "samples": len(sm),
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle alone
# ---------------------------------------------------------------------------

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    specs = q8gen.decode_matrices_05b()
    weights, xs = [], []
    for spec in specs:
        g, x = q8gen.q8_matrix(spec.seed, spec.M, spec.K, 1)
        weights.append((spec, g))
        xs.append(x)
    per_step_s = max(5.0, 60.0 / max(1, args.steps + args.warmup))
    rates = []
    for i in range(args.warmup + args.steps):
        r, tokens, dt, threads = oracle_decode_tokens(weights, xs, target_s=per_step_s)
        if i >= args.warmup:
            rates.append(r)
    value = statistics.median(rates)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tok/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 / value, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "batch": 1},
        "cpu_baseline": {"value": round(value, 3), "unit": "tok/s", "cores": threads,
                         "kind": "oracle",
                         "sample": f"whole decode tokens repeated for >= {per_step_s:.0f} s per step"},
        "e2e": {"value": round(value, 3), "unit": "tok/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", torch.cuda.current_device())

    from q8_block_quantized_02_b200 import build as q8build
    q8build.build()
    import q8_block_quantized_02_b200 as q8

    # ---- weights and activations (synthetic, resident in HBM) ----
    specs = q8gen.decode_matrices_05b()
    host_weights, host_x = [], []
    packed, x_off, y_bufs = [], [], []
    x_total = sum(s.K for s in specs)
    x_host = torch.empty(x_total, dtype=torch.float32).pin_memory()
    off = 0
    for spec in specs:
        g, x = q8gen.q8_matrix(spec.seed, spec.M, spec.K, 1)
        host_weights.append((spec, g))
        host_x.append(x)
        gd = torch.from_numpy(g).to(dev)
        p = torch.empty(q8.q8_packed_bytes(spec.M, spec.K), dtype=torch.uint8, device=dev)
        q8.q8_pack_weights(gd, spec.M, spec.K, p)
        del gd
        packed.append(p)
        x_host[off:off + spec.K] = torch.from_numpy(x[0])
        x_off.append(off)
        off += spec.K
        rows = spec.M // 2 if spec.swiglu else spec.M
        y_bufs.append(torch.empty(rows, dtype=torch.float32, device=dev))
    x_dev = x_host.to(dev)
    torch.cuda.synchronize()
    step_bytes = sum(algorithmic_bytes(s.M, s.K) for s in specs)

    def launch_one(i, stream):
        spec = specs[i]
        xv = x_dev[x_off[i]:x_off[i] + spec.K]
        if spec.swiglu:
            q8.q8_gate_up_swiglu(packed[i], xv, y_bufs[i], spec.M // 2, spec.K, 1, stream=stream)
        else:
            q8.q8_gemv(packed[i], xv, y_bufs[i], spec.M, spec.K, 1, stream=stream)

    def launch_step(stream):
        for i in range(len(specs)):
            launch_one(i, stream)

    lm = len(specs) - 1
    # kernel classes of the step: each is also captured on its own, its launches
    # back to back in step order (the same dependent PDL chain), to time the
    # kernel's average launch duration without other kernels in between
    classes = {
        "q8_gemv_n1": [i for i, s in enumerate(specs) if not s.swiglu and i != lm],
        "q8_gate_up_swiglu_n1": [i for i, s in enumerate(specs) if s.swiglu],
        "q8_gemv_n1_lm_head": [lm] * 4,
    }

    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        for _ in range(2):                     # eager warm-up (device setup happens here)
            launch_step(stream)
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            launch_step(stream)
        class_graphs = {}
        for name, idx in classes.items():
            cg = torch.cuda.CUDAGraph()
            with torch.cuda.graph(cg, stream=stream):
                for i in idx:
                    launch_one(i, stream)
            class_graphs[name] = cg
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()

    # CUDAGraph.replay() launches on torch's current stream: make it `stream`
    # for every replay below, so the events bracket exactly those launches.
    torch.cuda.set_stream(stream)

    # ---- warm-up replays ----
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()

    # ---- timed region: K steps of the captured decode token ----
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for _ in range(args.steps):
        graph.replay()
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    elapsed = max_over_ranks(t_start.elapsed_time(t_end) / 1e3, world, dev)

    # ---- per-kernel launch duration: each class's chain replayed on its own ----
    reps = max(10, min(100, args.steps // 20))
    kstats = {}
    for name, idx in classes.items():
        cg = class_graphs[name]
        for _ in range(3):
            cg.replay()
        torch.cuda.synchronize()
        k0 = torch.cuda.Event(enable_timing=True)
        k1 = torch.cuda.Event(enable_timing=True)
        k0.record(stream)
        for _ in range(reps):
            cg.replay()
        k1.record(stream)
        torch.cuda.synchronize()
        t_launch = k0.elapsed_time(k1) / 1e3 / (reps * len(idx))
        b_launch = sum(algorithmic_bytes(specs[i].M, specs[i].K) for i in idx) / len(idx)
        kstats[name] = {"launches_per_step": len(set(idx)), "avg_launch_us": t_launch * 1e6,
                        "bytes_per_launch": b_launch, "GBps": b_launch / t_launch / 1e9}

    # ---- end to end: host input -> device -> step -> host logits, per token ----
    logits_host = torch.empty(y_bufs[lm].numel(), dtype=torch.float32).pin_memory()
    e2e_steps = max(20, min(args.steps, 500))
    barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        x_dev.copy_(x_host, non_blocking=True)
        graph.replay()
        logits_host.copy_(y_bufs[lm], non_blocking=True)
        stream.synchronize()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_elapsed = max_over_ranks(e0.elapsed_time(e1) / 1e3, world, dev)

    # ---- CPU oracle baseline (rank 0, single GPU only) ----
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r, tokens, dt, threads = oracle_decode_tokens(host_weights, host_x, target_s=args.cpu_seconds)
        cpu = {"value": round(r, 3), "unit": "tok/s", "cores": threads, "kind": "oracle",
               "sample": f"{tokens} whole decode tokens (97 matrices each) in {dt:.1f} s, "
                         f"fp64 C oracle, OpenMP over output rows"}

    if world > 1:
        graph.reset()
        for cg in class_graphs.values():
            cg.reset()
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peak, peak_kind = measured_hbm_peak()
    tok_s = replica_throughput(world, args.steps, elapsed)
    gbs = step_bytes * args.steps / elapsed / 1e9  # per GPU
    dom = kstats["q8_gemv_n1"]
    achieved = dom["GBps"]
    line = {
        "metric": METRIC,
        "value": round(tok_s, 2),
        "unit": "tok/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(elapsed / args.steps * 1e3, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": {
            "workload": WORKLOAD,
            "batch": 1,
            "launches_per_step": len(specs),
            "weight_bytes_per_step": step_bytes,
            "l2": "no flush: 525 MB of weights per step, > 126 MB L2",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
        },
        "hbm_gbs_per_gpu": round(gbs, 1),
        "hbm_pct_of_8tbs": round(100 * gbs / NOMINAL_HBM_GBS, 2),
        "hbm_pct_of_measured_copy": round(100 * gbs / peak, 2),
        "roofline": {
            "kernel": "resident_kernel<1, fp32> (q8_gemv N=1 of qkv 1152x896, wo 896x896, down 896x4864)",
            "bound": "hbm",
            "achieved": round(achieved, 1),
            "peak": peak,
            "peak_kind": peak_kind,
            "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "traffic": None,
            "launches_per_step": dom["launches_per_step"],
            "bytes_per_launch": int(dom["bytes_per_launch"]),
            "avg_launch_us": round(dom["avg_launch_us"], 3),
            "timing": (f"CUDA events on the launch stream around {reps} replays of a graph holding "
                       f"this kernel's {dom['launches_per_step']} launches of a step, back to back"),
        },
        "kernels": {name: {"launches_per_step": k["launches_per_step"],
                           "avg_launch_us": round(k["avg_launch_us"], 3),
                           "bytes_per_launch": int(k["bytes_per_launch"]),
                           "GBps": round(k["GBps"], 1)} for name, k in kstats.items()},
        "e2e": {
            "value": round(replica_throughput(world, e2e_steps, e2e_elapsed), 2),
            "unit": "tok/s",
            "h2d_bytes_per_step": int(x_total * 4),
            "d2h_bytes_per_step": int(y_bufs[lm].numel() * 4),
            "steps": e2e_steps,
            "note": "pinned host x -> device, graph replay, logits -> pinned host, sync per token",
        },
        "gpu_launches": len(specs) * args.steps,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
