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
the CPU oracle timed on the host as a baseline (all cores and one thread),
and, under "configs", the device time per call of the other workloads (the
single 1152x896 GEMV, the 7B-class products at N = 1..16, the Qwen1.5-MoE
block at T = 1 and 8, the Q8 x Q8 sweep) with the oracle's time beside each.

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


TRAFFIC_PROFILE = os.path.join(ROOT, "profiles", "resident_gemv_decode_chain_qwen05b.md")


def measured_traffic():
    """DRAM bytes (read + write) per launch of the dominant kernel, from the
    committed ncu summary of the same kernel in the same decode chain (the
    line `traffic_bytes_per_launch: <n>`); None when there is none."""
    try:
        with open(TRAFFIC_PROFILE) as f:
            for line in f:
                if line.strip().startswith("traffic_bytes_per_launch:"):
                    return int(line.split(":", 1)[1].strip().split()[0])
    except (OSError, ValueError):
        pass
    return None


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
# the other workloads: one product per call, device time per call
# ---------------------------------------------------------------------------

def _graph_time_us(torch, stream, calls, replays=5):
    """Capture `calls` (a list of zero-argument launches on `stream`) in one
    CUDA graph, replay it, and return device microseconds per call (CUDA
    events on the launch stream around `replays` replays, after 2 untimed)."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for c in calls:
            c()
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(replays):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / (replays * len(calls))
    del g
    return us


def gpu_configs(q8, torch, dev, stream):
    """Device time per call of the single GEMV (1152x896, seed 0), the 7B-class
    small-batch products (N = 1, 2, 4, 8, 16 through the default entry points,
    N = 3, 4, 8, 16 through the split ones), the Qwen1.5-MoE block (T = 1, 8)
    the Q8 x Q8 sweep (M = 4096, K in {896, 3584, 4864, 18944}, N in {1,
    16}) and the K-quant GEMV on the 7B lm_head shape (Q4_K raw, Q6_K packed;
    N = 1, 2; block bytes 144 or 210 per 256 weights).  Calls walk distinct packed copies of each matrix covering several
    times the L2 (the same bytes, so only the cache behaviour differs), or
    distinct routings for the MoE block, so every call streams its weights
    from HBM.  Weight bytes are 34 per 32 weights."""
    import numpy as np
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    out = {}

    def packed_copies(g, M, K, min_bytes):
        nbytes = q8.q8_packed_bytes(M, K)
        n = max(1, int(np.ceil(min_bytes / nbytes)))
        src = torch.from_numpy(g).to(dev)
        ps = []
        for _ in range(n):
            p = torch.empty(nbytes, dtype=torch.uint8, device=dev)
            q8.q8_pack_weights(src, M, K, p, stream=stream)
            ps.append(p)
        del src
        return ps

    # single GEMV at the exact seed, rotated over >= 4 x L2 of copies
    M, K = 1152, 896
    g, x = q8gen.q8_matrix(0, M, K, 1)
    ps = packed_copies(g, M, K, 4 * l2)
    xd = torch.from_numpy(x).to(dev)
    y = torch.empty((1, M), dtype=torch.float32, device=dev)
    us = _graph_time_us(torch, stream, [lambda p=p: q8.q8_gemv(p, xd, y, M, K, 1, stream=stream) for p in ps])
    out["gemv_1152x896_n1_seed0"] = {"us_per_call": round(us, 3),
                                     "weight_GBps": round(algorithmic_bytes(M, K) / us / 1e3, 1),
                                     "rotation": f"{len(ps)} packed copies ({len(ps) * q8.q8_packed_bytes(M, K) >> 20} MiB)"}
    del ps

    # 7B-class small-batch products
    for spec in q8gen.small_batch_matrices_7b():
        g, _ = q8gen.q8_matrix(spec.seed, spec.M, spec.K)
        ps = packed_copies(g, spec.M, spec.K, 2 * l2)
        rows = spec.M // 2 if spec.swiglu else spec.M
        res = {}
        # the default entry point (CUDA cores) at every N; the split entry
        # point (tensor cores where faster) from N = 3
        for N, split in [(n, False) for n in (1, 2, 4, 8, 16)] + [(n, True) for n in (3, 4, 8, 16)]:
            xd = torch.from_numpy(q8gen.activations(100 + N, N, spec.K)).to(dev)
            y = torch.empty((N, rows), dtype=torch.float32, device=dev)
            if spec.swiglu:
                fn = q8.q8_gate_up_swiglu_split if split else q8.q8_gate_up_swiglu
                calls = [lambda p=p, fn=fn: fn(p, xd, y, rows, spec.K, N, stream=stream) for p in ps]
            else:
                fn = q8.q8_gemv_split if split else q8.q8_gemv
                calls = [lambda p=p, fn=fn: fn(p, xd, y, spec.M, spec.K, N, stream=stream) for p in ps]
            us = _graph_time_us(torch, stream, calls * max(1, 4 // len(ps)))
            res[f"N={N}" + (",split" if split else "")] = {
                "us_per_call": round(us, 2), "weight_GBps": round(algorithmic_bytes(spec.M, spec.K) / us / 1e3, 1)}
        key = f"7b_{spec.name}_{spec.M}x{spec.K}" + ("_swiglu" if spec.swiglu else "")
        out[key] = res
        del ps

    # Qwen1.5-MoE block: 60 experts + shared expert, top-4, cycling 16 routings
    E, H, I, Is, k = 60, 2048, 1408, 5632, 4

    def stack(seed0, n, Mx, Kx):
        one = q8.q8_packed_bytes(Mx, Kx)
        buf = torch.empty(n * one, dtype=torch.uint8, device=dev)
        for e in range(n):
            ge, _ = q8gen.q8_matrix(seed0 + e, Mx, Kx)
            q8.q8_pack_weights(torch.from_numpy(ge).to(dev), Mx, Kx, buf[e * one:(e + 1) * one], stream=stream)
        return buf

    p_gu, p_dn = stack(0, E, 2 * I, H), stack(1000, E, H, I)
    p_sgu, p_sdn = stack(E, 1, 2 * Is, H), stack(1000 + E, 1, H, Is)
    per_expert = (2 * I * H + H * I) * 34 // 32
    shared = (2 * Is * H + H * Is) * 34 // 32
    for T in (1, 8):
        R = 16
        idx = torch.empty((R, T, k), dtype=torch.int32, device=dev)
        w = torch.empty((R, T, k), dtype=torch.float32, device=dev)
        for r in range(R):
            lg = torch.from_numpy(q8gen.logits(61 + 100 * T + r, T, E)).to(dev)
            q8.q8_moe_route(lg, T, E, k, 0, idx[r], w[r], stream=stream)
        xd = torch.from_numpy(q8gen.activations(61, T, H)).to(dev)
        y = torch.empty((T, H), dtype=torch.float32, device=dev)
        ws_bytes = q8.q8_moe_workspace_bytes(T, E, k, H, I, Is)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        q8.q8_moe_workspace_init(ws, ws_bytes, stream=stream)
        calls = [lambda r=r: q8.q8_moe_gemv(p_gu, p_dn, p_sgu, p_sdn, idx[r], w[r], xd, y, T, E, k, H, I, Is,
                                            ws, ws_bytes, stream=stream) for r in range(R)]
        us = _graph_time_us(torch, stream, calls)
        picks = idx.cpu().numpy()
        mean_bytes = float(np.mean([len(np.unique(picks[r])) for r in range(R)])) * per_expert + shared
        out[f"moe_qwen1.5_a2.7b_T{T}"] = {"us_per_call": round(us, 2), "weight_MB_per_call": round(mean_bytes / 1e6, 2),
                                          "weight_GBps": round(mean_bytes / us / 1e3, 1),
                                          "rotation": f"{R} routings of N(0,1) logits, cycled"}
    del p_gu, p_dn, p_sgu, p_sdn

    # Q8 x Q8: quantise the activations (timed on its own), then the integer product
    M = 4096
    q8q8 = {}
    for K in (896, 3584, 4864, 18944):
        g, _ = q8gen.q8_matrix(K, M, K)
        ps = packed_copies(g, M, K, 4 * l2)
        for N in (1, 16):
            xf = torch.from_numpy(q8gen.activations(K + N, N, K)).to(dev)
            xq = torch.empty((N, K), dtype=torch.int8, device=dev)
            xd = torch.empty((N, K // 32), dtype=torch.int16, device=dev)
            y = torch.empty((N, M), dtype=torch.float32, device=dev)
            us_q = _graph_time_us(torch, stream, [lambda: q8.q8_quantize_act(xf, xq, xd, N, K, stream=stream)] * 20)
            us = _graph_time_us(torch, stream, [lambda p=p: q8.q8q8_gemv(p, xq, xd, y, M, K, N, stream=stream)
                                                for p in ps])
            q8q8[f"K={K},N={N}"] = {"us_per_call": round(us, 3), "quantize_us": round(us_q, 3),
                                    "weight_GBps": round(algorithmic_bytes(M, K) / us / 1e3, 1)}
        del ps
    out["q8q8_m4096"] = q8q8

    # K-quant GEMV (f3) on the 7B lm_head shape: Q4_K on its raw blocks, Q6_K
    # from its packed units; one copy of each (306 / 447 MB) exceeds the L2
    M, K = 152064, 3584
    for fmt, name in (("q4_k", "q4k"), ("q6_k", "q6k_packed")):
        blocks = torch.from_numpy(q8gen.kquant_matrix(fmt, 777, M, K)).to(dev)
        if fmt == "q6_k":
            w8 = torch.empty(q8.q8_q6k_packed_bytes(M, K), dtype=torch.uint8, device=dev)
            q8.q8_q6k_pack_weights(blocks, M, K, w8, stream=stream)
            fn = q8.q8_q6k_gemv_packed
        else:
            w8 = blocks
            fn = q8.q8_q4k_gemv
        kq = {}
        for N in (1, 2):
            xd = torch.from_numpy(q8gen.activations(778 + N, N, K)).to(dev)
            y = torch.empty((N, M), dtype=torch.float32, device=dev)
            us = _graph_time_us(torch, stream, [lambda: fn(w8, xd, y, M, K, N, stream=stream)] * 4)
            kq[f"N={N}"] = {"us_per_call": round(us, 2), "block_GBps": round(blocks.numel() / us / 1e3, 1)}
        out[f"7b_lm_head_{M}x{K}_{name}"] = kq
        del blocks, w8
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def oracle_configs(threads):
    """The fp64 CPU oracle on the same workloads (all host cores, OpenMP over
    output rows), each on a bounded sample: the whole single GEMV and MoE
    block; 128 rows of the large matrices, scaled to the full row count."""
    import oracle
    out = {}

    def timed(fn, min_s=0.3):
        n, t0 = 0, time.perf_counter()
        while True:
            fn()
            n += 1
            dt = time.perf_counter() - t0
            if dt >= min_s:
                return dt / n * 1e6

    g, x = q8gen.q8_matrix(0, 1152, 896, 1)
    out["gemv_1152x896_n1_seed0"] = {"oracle_us_per_call": round(timed(lambda: oracle.gemv(g, x, 1152, 896, threads=threads)), 1),
                                     "oracle_sample": "whole matrix"}
    S = 128
    for spec in q8gen.small_batch_matrices_7b():
        g, _ = q8gen.q8_matrix(spec.seed, S if not spec.swiglu else 2 * S, spec.K)
        res = {}
        for N in (1, 16):
            xs = q8gen.activations(100 + N, N, spec.K)
            if spec.swiglu:
                us = timed(lambda: oracle.gate_up_swiglu(g, xs, S, spec.K, threads=threads)) * (spec.M // 2) / S
            else:
                us = timed(lambda: oracle.gemv(g, xs, S, spec.K, threads=threads)) * spec.M / S
            res[f"N={N}"] = round(us, 1)
        key = f"7b_{spec.name}_{spec.M}x{spec.K}" + ("_swiglu" if spec.swiglu else "")
        out[key] = {"oracle_us_per_call": res, "oracle_sample": f"{S} output rows, scaled to {spec.M // (2 if spec.swiglu else 1)}"}
    E, H, I, Is, k = 60, 2048, 1408, 5632, 4
    gu, dn, sgu, sdn = q8gen.moe_weights(E, H, I, Is)
    for T in (1, 8):
        lg = q8gen.logits(61 + 100 * T, T, E)
        idx, w = oracle.route(lg, k)
        xs = q8gen.activations(61, T, H)
        us = timed(lambda: oracle.moe(gu, dn, sgu, sdn, idx, w, xs, H, I, Is, threads=threads), 0.5)
        out[f"moe_qwen1.5_a2.7b_T{T}"] = {"oracle_us_per_call": round(us, 1), "oracle_sample": "whole block"}
    q = {}
    for K in (896, 3584, 4864, 18944):
        g, _ = q8gen.q8_matrix(K, S, K)
        for N in (1, 16):
            xq, xd, _ = oracle.quantize_act(q8gen.activations(K + N, N, K))
            q[f"K={K},N={N}"] = round(timed(lambda: oracle.q8q8(g, xq, xd, S, K, want_dots=False, threads=threads))
                                      * 4096 / S, 1)
    out["q8q8_m4096"] = {"oracle_us_per_call": q, "oracle_sample": f"{S} output rows, scaled to 4096"}
    for fmt, name in (("q4_k", "q4k"), ("q6_k", "q6k_packed")):
        blocks = q8gen.kquant_matrix(fmt, 777, S, 3584)
        res = {}
        for N in (1, 2):
            xs = q8gen.activations(778 + N, N, 3584)
            res[f"N={N}"] = round(timed(lambda: oracle.kquant_gemv(fmt, blocks, xs, S, 3584, threads=threads))
                                  * 152064 / S, 1)
        out[f"7b_lm_head_152064x3584_{name}"] = {"oracle_us_per_call": res,
                                                 "oracle_sample": f"{S} output rows (raw blocks), scaled to 152064"}
    return out


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

    # ---- the other workloads, one product per call (single GPU only) ----
    configs = None
    if world == 1 and not args.no_configs:
        with torch.cuda.stream(stream):
            configs = gpu_configs(q8, torch, dev, stream)

    # ---- CPU oracle baseline (rank 0, single GPU only): all host cores and
    # one thread, the row split across threads of "Lumen v0.3.0" Phase 7.J ----
    cpu = cpu1 = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r, tokens, dt, threads = oracle_decode_tokens(host_weights, host_x, target_s=args.cpu_seconds)
        cpu = {"value": round(r, 3), "unit": "tok/s", "cores": threads, "kind": "oracle",
               "sample": f"{tokens} whole decode tokens (97 matrices each) in {dt:.1f} s, "
                         f"fp64 C oracle, OpenMP over output rows"}
        r1, tokens1, dt1, _ = oracle_decode_tokens(host_weights, host_x, target_s=args.cpu_seconds, threads=1)
        cpu1 = {"value": round(r1, 3), "unit": "tok/s", "cores": 1, "kind": "oracle",
                "sample": f"{tokens1} whole decode tokens (97 matrices each) in {dt1:.1f} s, fp64 C oracle"}
        if configs is not None:
            for key, v in oracle_configs(threads).items():
                configs.setdefault(key, {}).update(v)

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
            "traffic": measured_traffic(),
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
        "cpu_baseline_1thread": cpu1,
        "configs": configs,
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
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads (single GEMV, 7B small batch, MoE, Q8 x Q8)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
