"""Run one libq8 product on synthetic Qwen-shaped inputs and time it.

    python -m q8_block_quantized_02_b200.profile --op gemv --M 151936 --K 896 --N 1
    python -m q8_block_quantized_02_b200.profile --op q8q8 --M 37888 --K 3584 --N 16
    python -m q8_block_quantized_02_b200.profile --op argmax --M 151936 --K 896 --N 1
    python -m q8_block_quantized_02_b200.profile --op moe --T 1
    python -m q8_block_quantized_02_b200.profile --op readpeak
    python -m q8_block_quantized_02_b200.profile --op decode --reps 3

Weights follow the synthetic Q8_0 recipe (q uniform in [-127, 127], d =
|N(0,1)| * 0.02) and activations are N(0,1).  Enough packed copies of the
weight matrix are made to cover three times the L2 cache, and the calls walk
through them, so every timed call streams its weights from HBM.  Each call is
one launch of the library's kernel on the current stream; the time per call
comes from CUDA events around `--reps` back-to-back calls after `--warmup`
untimed ones.  Prints one JSON line with microseconds per call and the weight
bytes (34 per 32 weights) per second.

This is also the driver for ncu captures of a single kernel: with
`--copies 1 --reps 3 --warmup 2` it makes five launches on one matrix.

`--op moe` times q8_moe_gemv on Qwen1.5-MoE-A2.7B shapes (60 experts of
gate_up 2816 x 2048 and down 2048 x 1408, a shared expert of intermediate
5632, top-4; all sizes can be changed).  All experts are packed once
(about 590 MB, more than L2).  `--routings` sets of router logits ~ N(0,1)
are routed up front (q8_moe_route, not timed) and the timed calls cycle
through them, so consecutive calls select different experts.  Bytes per
call count each call's distinct selected experts plus the shared expert once
(34 B per 32 weights).

`--op decode` runs `--reps` decode steps of the Qwen2.5-0.5B matmul set (the
benchmark's step: 24 x {qkv, wo, gate_up + SwiGLU, down} + lm_head, 97
dependent launches on one stream), eagerly, after `--warmup` steps: the
driver of ncu captures of the decode kernels in their chain.

`--op readpeak` is a reference figure, not a libq8 product: the HBM read rate
of a plain reduction (torch.sum over 4 GiB of fp32, so every byte is read
once and nothing is written back), the read-only counterpart of the measured
copy peak.
"""
from __future__ import annotations

import argparse
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--op", choices=["gemv", "argmax", "swiglu", "q8q8", "q4k", "q6k", "q6kp", "moe", "readpeak",
                             "decode"],
                    default="gemv",
                    help="q8_gemv, q8_gemv_argmax (logits not written), q8_gate_up_swiglu (M = rows of "
                         "the stacked gate|up matrix) or q8_quantize_act + q8q8_gemv (only q8q8_gemv is "
                         "timed)")
    ap.add_argument("--M", type=int, default=151936)
    ap.add_argument("--K", type=int, default=896)
    ap.add_argument("--N", type=int, default=1)
    ap.add_argument("--reps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--copies", type=int, default=0, help="packed weight copies (0: cover 3x L2)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--split", action="store_true",
                    help="gemv / swiglu: the _split entry points (tensor cores where they serve)")
    ap.add_argument("--T", type=int, default=1, help="moe: tokens")
    ap.add_argument("--E", type=int, default=60, help="moe: routed experts")
    ap.add_argument("--H", type=int, default=2048, help="moe: hidden size")
    ap.add_argument("--I", type=int, default=1408, help="moe: expert intermediate size")
    ap.add_argument("--Is", type=int, default=5632, help="moe: shared expert intermediate size (0: none)")
    ap.add_argument("--k", type=int, default=4, help="moe: experts per token")
    ap.add_argument("--routings", type=int, default=16, help="moe: distinct routings cycled through")
    args = ap.parse_args(argv)
    if args.op == "moe":
        return _moe(args)
    if args.op == "readpeak":
        return _readpeak(args)
    if args.op == "decode":
        return _decode(args)

    import numpy as np
    import torch

    import q8gen
    import q8_block_quantized_02_b200 as q8

    M, K, N = args.M, args.K, args.N
    dev = torch.device("cuda", torch.cuda.current_device())
    if args.op in ("q4k", "q6k", "q6kp"):
        return _kquant(args, q8, q8gen, np, torch, dev)
    g, x = q8gen.q8_matrix(args.seed, M, K, N)
    nbytes = q8.q8_packed_bytes(M, K)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    copies = args.copies if args.copies > 0 else max(1, int(np.ceil(3 * l2 / nbytes)))
    src = torch.from_numpy(g).to(dev)
    packs = []
    for _ in range(copies):
        p = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        q8.q8_pack_weights(src, M, K, p)
        packs.append(p)
    del src
    xf = torch.from_numpy(x).to(dev)
    if args.op == "swiglu":
        if M % 16:
            raise SystemExit("--op swiglu needs M = 2 * I with I % 8 == 0")
        y = torch.empty((N, M // 2), dtype=torch.float32, device=dev)
    else:
        y = torch.empty((N, M), dtype=torch.float32, device=dev)
    if args.op == "argmax":
        best = torch.empty((N,), dtype=torch.int64, device=dev)
    if args.op == "q8q8":
        xq = torch.empty((N, K), dtype=torch.int8, device=dev)
        xd = torch.empty((N, K // 32), dtype=torch.int16, device=dev)
        q8.q8_quantize_act(xf, xq, xd, N, K)

    it = [0]

    def call():
        p = packs[it[0] % copies]
        it[0] += 1
        if args.op == "gemv":
            (q8.q8_gemv_split if args.split else q8.q8_gemv)(p, xf, y, M, K, N)
        elif args.op == "argmax":
            q8.q8_gemv_argmax(p, xf, None, M, K, N, best)
        elif args.op == "swiglu":
            if args.split:
                q8.q8_gate_up_swiglu_split(p, xf, y, M // 2, K, N)
            else:
                q8.q8_gate_up_swiglu(p, xf, y, M // 2, K, N)
        else:
            q8.q8q8_gemv(p, xq, xd, y, M, K, N)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.reps):
        call()
    t1.record()
    torch.cuda.synchronize()
    st, word = q8.q8_read_device_error()
    us = t0.elapsed_time(t1) * 1e3 / max(1, args.reps)
    weight_bytes = M * K * 34 // 32
    print(json.dumps({"op": args.op, "M": M, "K": K, "N": N, "us_per_call": round(us, 3),
                      "weight_GBps": round(weight_bytes / (us * 1e-6) / 1e9, 1), "copies": copies,
                      "reps": args.reps, "device_error": word}), flush=True)
    return 0 if st == 0 else 1


def _kquant(args, q8, q8gen, np, torch, dev) -> int:
    """q8_q4k_gemv / q8_q6k_gemv on raw GGUF K-quant blocks (random fields), or
    q8_q6k_gemv_packed (q6kp) on their packed units; bytes per call are the
    blocks' (144 or 210 per 256 weights)."""
    M, K, N = args.M, args.K, args.N
    fmt = "q4_k" if args.op == "q4k" else "q6_k"
    blocks = q8gen.kquant_matrix(fmt, args.seed, M, K)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    copies = args.copies if args.copies > 0 else max(1, int(np.ceil(3 * l2 / blocks.size)))
    src = torch.from_numpy(blocks).to(dev)
    if args.op == "q6kp":
        ws = []
        for _ in range(copies):
            p = torch.empty(q8.q8_q6k_packed_bytes(M, K), dtype=torch.uint8, device=dev)
            q8.q8_q6k_pack_weights(src, M, K, p)
            ws.append(p)
    else:
        ws = [src.clone() for _ in range(copies)]
    del src
    x = torch.from_numpy(q8gen.activations(args.seed + 1, N, K)).to(dev)
    y = torch.empty((N, M), dtype=torch.float32, device=dev)
    fn = {"q4k": q8.q8_q4k_gemv, "q6k": q8.q8_q6k_gemv, "q6kp": q8.q8_q6k_gemv_packed}[args.op]
    for i in range(args.warmup):
        fn(ws[i % copies], x, y, M, K, N)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(args.reps):
        fn(ws[i % copies], x, y, M, K, N)
    t1.record()
    torch.cuda.synchronize()
    st, word = q8.q8_read_device_error()
    us = t0.elapsed_time(t1) * 1e3 / max(1, args.reps)
    print(json.dumps({"op": args.op, "M": M, "K": K, "N": N, "us_per_call": round(us, 3),
                      "weight_GBps": round(blocks.size / (us * 1e-6) / 1e9, 1), "copies": copies,
                      "reps": args.reps, "device_error": word}), flush=True)
    return 0 if st == 0 else 1


def _decode(args) -> int:
    import torch

    import q8gen
    import q8_block_quantized_02_b200 as q8

    dev = torch.device("cuda", torch.cuda.current_device())
    specs = q8gen.decode_matrices_05b()
    packed, xs, ys = [], [], []
    for s in specs:
        g, x = q8gen.q8_matrix(s.seed, s.M, s.K, 1)
        p = torch.empty(q8.q8_packed_bytes(s.M, s.K), dtype=torch.uint8, device=dev)
        q8.q8_pack_weights(torch.from_numpy(g).to(dev), s.M, s.K, p)
        packed.append(p)
        xs.append(torch.from_numpy(x[0]).to(dev))
        ys.append(torch.empty(s.M // 2 if s.swiglu else s.M, dtype=torch.float32, device=dev))

    def step():
        for i, s in enumerate(specs):
            if s.swiglu:
                q8.q8_gate_up_swiglu(packed[i], xs[i], ys[i], s.M // 2, s.K, 1)
            else:
                q8.q8_gemv(packed[i], xs[i], ys[i], s.M, s.K, 1)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.reps):
        step()
    t1.record()
    torch.cuda.synchronize()
    st, word = q8.q8_read_device_error()
    us = t0.elapsed_time(t1) * 1e3 / max(1, args.reps)
    print(json.dumps({"op": "decode", "launches_per_step": len(specs), "us_per_step_eager": round(us, 2),
                      "reps": args.reps, "device_error": word}), flush=True)
    return 0 if st == 0 else 1


def _readpeak(args) -> int:
    import torch

    dev = torch.device("cuda", torch.cuda.current_device())
    n = (4 << 30) // 4
    a = torch.ones(n, dtype=torch.float32, device=dev)
    out = torch.empty((), dtype=torch.float32, device=dev)
    for _ in range(max(3, args.warmup)):
        torch.sum(a, 0, out=out)
    torch.cuda.synchronize()
    reps = max(5, min(args.reps, 50))
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(reps):
        torch.sum(a, 0, out=out)
    t1.record()
    torch.cuda.synchronize()
    us = t0.elapsed_time(t1) * 1e3 / reps
    assert abs(float(out.item()) - n) <= 1e-3 * n
    print(json.dumps({"op": "readpeak", "bytes": n * 4, "us_per_call": round(us, 2),
                      "read_GBps": round(n * 4 / (us * 1e-6) / 1e9, 1), "reps": reps}), flush=True)
    return 0


def _moe(args) -> int:
    import numpy as np
    import torch

    import q8gen
    import q8_block_quantized_02_b200 as q8

    T, E, H, I, Is, k = args.T, args.E, args.H, args.I, args.Is, args.k
    dev = torch.device("cuda", torch.cuda.current_device())

    def stack(seed0, n, M, K):
        one = q8.q8_packed_bytes(M, K)
        out = torch.empty(n * one, dtype=torch.uint8, device=dev)
        for e in range(n):
            g, _ = q8gen.q8_matrix(seed0 + e, M, K)
            q8.q8_pack_weights(torch.from_numpy(g).to(dev), M, K, out[e * one:(e + 1) * one])
        return out

    p_gu, p_dn = stack(args.seed, E, 2 * I, H), stack(args.seed + 1000, E, H, I)
    p_sgu = p_sdn = None
    if Is:
        p_sgu, p_sdn = stack(args.seed + 2000, 1, 2 * Is, H), stack(args.seed + 2001, 1, H, Is)
    R = max(1, args.routings)
    idx = torch.empty((R, T, k), dtype=torch.int32, device=dev)
    w = torch.empty((R, T, k), dtype=torch.float32, device=dev)
    for r in range(R):
        lg = torch.from_numpy(q8gen.logits(args.seed + 100 + r, T, E)).to(dev)
        q8.q8_moe_route(lg, T, E, k, 0, idx[r], w[r])
    x = torch.from_numpy(q8gen.activations(args.seed + 7, T, H)).to(dev)
    y = torch.empty((T, H), dtype=torch.float32, device=dev)
    ws_bytes = q8.q8_moe_workspace_bytes(T, E, k, H, I, Is)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    q8.q8_moe_workspace_init(ws, ws_bytes)
    it = [0]

    def call():
        r = it[0] % R
        it[0] += 1
        q8.q8_moe_gemv(p_gu, p_dn, p_sgu, p_sdn, idx[r], w[r], x, y, T, E, k, H, I, Is, ws, ws_bytes)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    start = it[0]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.reps):
        call()
    t1.record()
    torch.cuda.synchronize()
    st, word = q8.q8_read_device_error()
    us = t0.elapsed_time(t1) * 1e3 / max(1, args.reps)
    per_expert = (2 * I * H + H * I) * 34 // 32
    shared = (2 * Is * H + H * Is) * 34 // 32
    picks = idx.cpu().numpy()
    uniq = [len(np.unique(picks[(start + i) % R])) for i in range(args.reps)]
    mean_bytes = float(np.mean(uniq)) * per_expert + shared
    print(json.dumps({"op": "moe", "T": T, "E": E, "H": H, "I": I, "Is": Is, "k": k,
                      "us_per_call": round(us, 3), "unique_experts": round(float(np.mean(uniq)), 2),
                      "weight_MB": round(mean_bytes / 1e6, 2),
                      "weight_GBps": round(mean_bytes / (us * 1e-6) / 1e9, 1), "routings": R,
                      "reps": args.reps, "device_error": word}), flush=True)
    return 0 if st == 0 else 1


if __name__ == "__main__":
    raise SystemExit(main())
