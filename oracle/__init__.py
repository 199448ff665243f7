"""CPU oracle for the Q8_0 decode-product hot path (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  It wraps ``q8_oracle.c`` -- plain C, fp64
accumulation, no code shared with the CUDA library -- through ctypes, and
builds it with gcc on first use.  Every function takes and returns numpy
arrays; GGUF weights are raw Q8_0 bytes (34 bytes per 32 weights: a
little-endian binary16 scale, then 32 int8), as the "skuznetsov/cogni-ml"
README's Q8_0 GEMV probe reads them ("Build Qwen CLIs").

Parity of this oracle is pinned by ``tests/test_oracle_pins.py`` (closed forms,
brute force with exact rationals, linearity, round trip, hand-computed blocks,
library conversions).  The only unpinned quantity is the fp64 rounding order
of large sums, which the GPU tolerance dwarfs.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "q8_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

QK = 32
BLOCK_BYTES = 34

_P = ctypes.c_void_p
_I64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile q8_oracle.c into liboracle.so (gcc, -O2 -ffp-contract=off, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-std=c11",
           "-Wall", "-Wextra", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_half_to_double.restype = ctypes.c_double
        lib.oracle_float_to_half_rn.argtypes = [ctypes.c_float]
        lib.oracle_float_to_half_rn.restype = ctypes.c_uint16
        lib.oracle_gemv.argtypes = [_P, _P, _I64, _I64, _I64, _P, _P, ctypes.c_int]
        lib.oracle_gemv.restype = None
        lib.oracle_gate_up_swiglu.argtypes = [_P, _P, _I64, _I64, _I64, _P, _P, _P, _P, _P,
                                              ctypes.c_int]
        lib.oracle_gate_up_swiglu.restype = None
        lib.oracle_route.argtypes = [_P, _I64, _I64, _I64, ctypes.c_int, _P, _P]
        lib.oracle_route.restype = ctypes.c_int
        lib.oracle_moe.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64,
                                   _I64, _P, _P, _P, ctypes.c_int]
        lib.oracle_moe.restype = None
        lib.oracle_quantize_act.argtypes = [_P, _I64, _I64, _P, _P, _P]
        lib.oracle_quantize_act.restype = None
        lib.oracle_q8q8.argtypes = [_P, _P, _P, _I64, _I64, _I64, _P, _P, _P, ctypes.c_int]
        lib.oracle_q8q8.restype = None
        lib.oracle_quantize_weights.argtypes = [_P, _I64, _I64, _P, _P]
        lib.oracle_quantize_weights.restype = None
        lib.oracle_kquant_gemv.argtypes = [ctypes.c_int, _P, _P, _I64, _I64, _I64, _P, _P, _P, ctypes.c_int]
        lib.oracle_kquant_gemv.restype = None
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = ctypes.c_int
        _lib = lib
        return lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _u8(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.uint8).reshape(-1)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


def max_threads() -> int:
    """Threads the oracle's OpenMP loops may use on this host."""
    return int(_load().oracle_max_threads())


def half_to_double(bits: int) -> float:
    """Value of a binary16 bit pattern (IEEE 754 definition)."""
    return float(_load().oracle_half_to_double(int(bits) & 0xFFFF))


def float_to_half_rn(value: float) -> int:
    """binary16 bits of an fp32 value, round to nearest even."""
    return int(_load().oracle_float_to_half_rn(float(np.float32(value))))


def gemv(gguf, x, M: int, K: int, N: int | None = None, threads: int = 1):
    """O1: y[n, m] = sum_k d*q[m, k] * x[n, k] in fp64.  Returns (y, y_abs) [N][M]."""
    x = _f32(x).reshape(-1, K)
    N = x.shape[0] if N is None else N
    g = _u8(gguf)
    assert g.size == M * (K // QK) * BLOCK_BYTES
    y = np.empty((N, M), np.float64)
    ya = np.empty((N, M), np.float64)
    _load().oracle_gemv(_ptr(g), _ptr(x), M, K, N, _ptr(y), _ptr(ya), int(threads))
    return y, ya


KQ_BYTES = {"q4_k": 144, "q6_k": 210}


def kquant_gemv(fmt: str, blocks, x, M: int, K: int, threads: int = 1, want_w: bool = False):
    """O11: y = W x in fp64 for a raw GGUF Q4_K or Q6_K matrix (the K-quant GEMV
    probes of the "skuznetsov/cogni-ml" README, "Build Qwen CLIs"); the block
    packing is written out in q8_oracle.c.  Returns (y, y_abs[, w]) with
    y_abs = sum_k |w x| and w the dequantised [M][K] weights."""
    x = _f32(x).reshape(-1, K)
    N = x.shape[0]
    b = _u8(blocks)
    assert K % 256 == 0 and b.size == M * (K // 256) * KQ_BYTES[fmt]
    y = np.empty((N, M), np.float64)
    ya = np.empty((N, M), np.float64)
    w = np.empty((M, K), np.float64) if want_w else None
    _load().oracle_kquant_gemv(4 if fmt == "q4_k" else 6, _ptr(b), _ptr(x), M, K, N, _ptr(y), _ptr(ya),
                               _ptr(w), int(threads))
    return (y, ya, w) if want_w else (y, ya)


def gemv_residual(gguf, x, residual, M: int, K: int, threads: int = 1):
    """O10: the O1 GEMV plus a residual stream, y + residual in fp64 (the
    residual add after the attention output and MLP down projections;
    "fusedtok 1.3.0" fused residual add).  Returns (y + residual, y_abs)."""
    y, ya = gemv(gguf, x, M, K, threads=threads)
    return y + np.asarray(residual, np.float64).reshape(y.shape), ya


def gemv_argmax(gguf, x, M: int, K: int, threads: int = 1):
    """O8: greedy pick after the O1 GEMV: for each activation row n, the index
    of the largest y[n, m], the lowest such index when several are equal (the
    resident top-1 step of the "skuznetsov/cogni-ml" README; earliest-index
    ties as in "fusedtok 1.3.0", "API stability").  Returns (idx [N] int64,
    y, y_abs) with y, y_abs from gemv()."""
    y, ya = gemv(gguf, x, M, K, threads=threads)
    # numpy's argmax returns the first occurrence of the maximum
    return np.argmax(y, axis=1).astype(np.int64), y, ya


def gate_up_swiglu(gguf, x, I: int, K: int, threads: int = 1):
    """O2: h = silu(g) * u with g = rows [0, I), u = rows [I, 2I) of W.

    Returns dict of fp64 [N][I] arrays: h, g, u, g_abs, u_abs."""
    x = _f32(x).reshape(-1, K)
    N = x.shape[0]
    g8 = _u8(gguf)
    assert g8.size == 2 * I * (K // QK) * BLOCK_BYTES
    out = {k: np.empty((N, I), np.float64) for k in ("h", "g", "u", "g_abs", "u_abs")}
    _load().oracle_gate_up_swiglu(_ptr(g8), _ptr(x), I, K, N, _ptr(out["h"]), _ptr(out["g"]),
                                  _ptr(out["u"]), _ptr(out["g_abs"]), _ptr(out["u_abs"]),
                                  int(threads))
    return out


def route(logits, top_k: int, renormalize: bool = False):
    """O3: softmax + top-k (ties to the lowest index).  Returns (idx int32, w fp64)."""
    logits = _f32(logits)
    T, E = logits.shape
    idx = np.empty((T, top_k), np.int32)
    w = np.empty((T, top_k), np.float64)
    rc = _load().oracle_route(_ptr(logits), T, E, top_k, int(bool(renormalize)), _ptr(idx),
                              _ptr(w))
    if rc != 0:
        raise ValueError("oracle_route: NaN logit" if rc == -1 else f"oracle_route rc={rc}")
    return idx, w


def moe(gate_up_all, down_all, shared_gate_up, shared_down, idx, w, x, H: int, I: int,
        I_shared: int, threads: int = 1):
    """O4: routed-expert MoE block plus shared expert (weight 1).

    gate_up_all / down_all: E consecutive GGUF matrices ([2I][H] / [H][I]).
    Returns (y, bound, slot_out) -- fp64 [T][H], [T][H], [T][k][H]."""
    x = _f32(x).reshape(-1, H)
    T = x.shape[0]
    idx = np.ascontiguousarray(idx, np.int32)
    w = np.ascontiguousarray(w, np.float64)
    k = idx.shape[1]
    gu = _u8(gate_up_all)
    dn = _u8(down_all)
    E = gu.size // (2 * I * (H // QK) * BLOCK_BYTES)
    sgu = _u8(shared_gate_up) if shared_gate_up is not None else None
    sdn = _u8(shared_down) if shared_down is not None else None
    y = np.empty((T, H), np.float64)
    bound = np.empty((T, H), np.float64)
    slot_out = np.empty((T, k, H), np.float64)
    _load().oracle_moe(_ptr(gu), _ptr(dn), _ptr(sgu), _ptr(sdn), _ptr(idx), _ptr(w), _ptr(x),
                       T, E, k, H, I, I_shared if sgu is not None else 0, _ptr(y), _ptr(bound),
                       _ptr(slot_out), int(threads))
    return y, bound, slot_out


def quantize_act(x, K: int | None = None):
    """O5: per-32-block activation quantisation.  Returns (q int8 [N][K],
    d binary16 bits uint16 [N][K/32], d32 fp32 [N][K/32])."""
    x = _f32(x)
    if K is None:
        K = x.shape[-1]
    x = x.reshape(-1, K)
    N = x.shape[0]
    q = np.empty((N, K), np.int8)
    d = np.empty((N, K // QK), np.uint16)
    d32 = np.empty((N, K // QK), np.float32)
    _load().oracle_quantize_act(_ptr(x), N, K, _ptr(q), _ptr(d), _ptr(d32))
    return q, d, d32


def rmsnorm_quantize_act(x, gamma, eps: float, r=None):
    """O9: RMSNorm then the O5 quantiser.  r_exact[n] = 1 / sqrt(mean_k x^2 +
    eps) in fp64 (the RMSNorm before every Qwen projection, "augur" README,
    "Features"; "fusedtok 1.3.0" rmsnorm(x, w, eps)).  The codes are taken
    from xhat = (x * r) * gamma with two fp32 roundings in that order, where r
    is the given fp32 per-row factor (the kernel's own; by default r_exact
    rounded to fp32), so a quantised code is decided in the kernel's
    precision.  Returns (r_exact fp64 [N], xhat fp32 [N][K], q, d, d32) with
    q, d, d32 from quantize_act(xhat)."""
    x = _f32(x).reshape(-1, np.asarray(gamma).size)
    gamma = _f32(gamma).reshape(-1)
    x64 = x.astype(np.float64)
    eps64 = float(np.float32(eps))
    r_exact = 1.0 / np.sqrt(np.mean(x64 * x64, axis=1) + eps64)
    r32 = r_exact.astype(np.float32) if r is None else _f32(r).reshape(-1)
    xhat = (x * r32[:, None]).astype(np.float32)          # fp32 product, round to nearest
    xhat = (xhat * gamma[None, :]).astype(np.float32)     # then the gain, another rounding
    q, d, d32 = quantize_act(xhat)
    return r_exact, xhat, q, d, d32


def q8q8(gguf, xq, xd, M: int, K: int, want_dots: bool = True, threads: int = 1):
    """O6: int32 block dots and y = sum_b d_w d_x dot_b (fp64).

    Returns (dots int32 [N][M][K/32] or None, y fp64 [N][M], y_abs fp64 [N][M])."""
    xq = np.ascontiguousarray(xq, np.int8).reshape(-1, K)
    N = xq.shape[0]
    xd = np.ascontiguousarray(xd, np.uint16).reshape(N, K // QK)
    g8 = _u8(gguf)
    dots = np.empty((N, M, K // QK), np.int32) if want_dots else None
    y = np.empty((N, M), np.float64)
    ya = np.empty((N, M), np.float64)
    _load().oracle_q8q8(_ptr(g8), _ptr(xq), _ptr(xd), M, K, N, _ptr(dots), _ptr(y), _ptr(ya),
                        int(threads))
    return dots, y, ya


def quantize_weights(w, K: int | None = None):
    """O7 (test aid): fp32 weights -> GGUF Q8_0 bytes with the O5 rule.

    Returns (gguf uint8 [M*K/32*34], d32 fp32 [M][K/32])."""
    w = _f32(w)
    if K is None:
        K = w.shape[-1]
    w = w.reshape(-1, K)
    M = w.shape[0]
    gguf = np.empty(M * (K // QK) * BLOCK_BYTES, np.uint8)
    d32 = np.empty((M, K // QK), np.float32)
    _load().oracle_quantize_weights(_ptr(w), M, K, _ptr(gguf), _ptr(d32))
    return gguf, d32
