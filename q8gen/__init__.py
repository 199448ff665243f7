"""Seeded synthetic inputs for the Q8_0 decode-product workloads.

This module is shared by the tests, the benchmark and the smoke check, and it
holds none of the method's arithmetic: it only draws random numbers and lays
the drawn values out as GGUF Q8_0 bytes (34 bytes per 32 weights: the
little-endian binary16 scale d, then 32 int8 values q).  Both the CUDA path and
the CPU oracle consume exactly these bytes.

Recipe (one numpy PCG64 generator per matrix, seeded with its own seed):
  1. q = integers(-127, 128, (M, K), int8)            uniform on [-127, 127]
  2. d = (|standard_normal((M, K/32))| * 0.02) -> float16 (round to nearest)
  3. x = standard_normal((N, K)) -> float32            (only when N is given)
Workload shapes are the Qwen-family shapes named below; there are no real
weights, prompts or datasets anywhere in this repository.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

QK = 32
BLOCK_BYTES = 34


def assemble_gguf(q: np.ndarray, d_bits: np.ndarray) -> np.ndarray:
    """Lay out int8 q [M][K] and binary16 bit patterns d [M][K/32] as GGUF Q8_0
    bytes [M][K/32][34] (flattened uint8)."""
    q = np.ascontiguousarray(q, np.int8)
    M, K = q.shape
    B = K // QK
    d_bits = np.ascontiguousarray(d_bits).view(np.uint16).reshape(M, B)
    out = np.empty((M, B, BLOCK_BYTES), np.uint8)
    out[:, :, 0] = (d_bits & 0xFF).astype(np.uint8)
    out[:, :, 1] = (d_bits >> 8).astype(np.uint8)
    out[:, :, 2:] = q.view(np.uint8).reshape(M, B, QK)
    return out.reshape(-1)


def split_gguf(gguf: np.ndarray, M: int, K: int):
    """Inverse of assemble_gguf: returns (q int8 [M][K], d_bits uint16 [M][K/32])."""
    b = np.ascontiguousarray(gguf, np.uint8).reshape(M, K // QK, BLOCK_BYTES)
    d_bits = b[:, :, 0].astype(np.uint16) | (b[:, :, 1].astype(np.uint16) << 8)
    q = np.ascontiguousarray(b[:, :, 2:]).view(np.int8).reshape(M, K)
    return q, d_bits


def q8_matrix(seed: int, M: int, K: int, N: int | None = None):
    """Draw one Q8_0 matrix (and optionally its activations) per the recipe.

    Returns (gguf uint8 bytes, x float32 [N][K] or None)."""
    if K % QK:
        raise ValueError("K must be a multiple of 32")
    rng = np.random.default_rng(seed)
    q = rng.integers(-127, 128, size=(M, K), dtype=np.int8)
    d = (np.abs(rng.standard_normal((M, K // QK))) * 0.02).astype(np.float16)
    gguf = assemble_gguf(q, d.view(np.uint16))
    x = rng.standard_normal((N, K)).astype(np.float32) if N is not None else None
    return gguf, x


KQ_BYTES = {"q4_k": 144, "q6_k": 210}


def kquant_matrix(fmt: str, seed: int, M: int, K: int) -> np.ndarray:
    """Raw GGUF K-quant bytes [M][K/256][144 or 210] (flattened uint8): every
    packed field is uniform random bytes, except the binary16 super-block
    scales, drawn as |N(0,1)| * 1e-4 (Q4_K d and dmin, bytes 0-3) or
    |N(0,1)| * 2e-5 (Q6_K d, bytes 208-209), so weights land near the Q8_0
    recipe's magnitude and some scales are subnormal."""
    if K % 256:
        raise ValueError("K must be a multiple of 256")
    rng = np.random.default_rng(seed)
    nb = M * (K // 256)
    b = rng.integers(0, 256, size=(nb, KQ_BYTES[fmt]), dtype=np.uint8)
    if fmt == "q4_k":
        dd = (np.abs(rng.standard_normal((nb, 2))) * 1e-4).astype(np.float16)
        b[:, 0:4] = dd.view(np.uint8).reshape(nb, 4)
    else:
        d = (np.abs(rng.standard_normal(nb)) * 2e-5).astype(np.float16)
        b[:, 208:210] = d.view(np.uint8).reshape(nb, 2)
    return b.reshape(-1)


def activations(seed: int, N: int, K: int) -> np.ndarray:
    """fp32 activations x [N][K] ~ N(0, 1) from their own generator."""
    return np.random.default_rng(seed).standard_normal((N, K)).astype(np.float32)


def logits(seed: int, T: int, E: int) -> np.ndarray:
    """fp32 router logits [T][E] ~ N(0, 1)."""
    return np.random.default_rng(seed).standard_normal((T, E)).astype(np.float32)


# --------------------------------------------------------------------------
# Workload shapes
# --------------------------------------------------------------------------

@dataclass(frozen=True)
class MatSpec:
    name: str
    M: int          # output rows (for a fused gate_up: 2 * I)
    K: int
    swiglu: bool    # fused gate_up + SiLU(gate) * up
    seed: int


# Qwen2.5-0.5B shapes: hidden 896, intermediate 4864, 24 layers,
# 14 q heads / 2 kv heads of dim 64 (qkv rows 896 + 2*128 = 1152), vocab 151936.
QWEN05B = dict(hidden=896, intermediate=4864, layers=24, qkv=1152, vocab=151936)

# 7B-class shapes: hidden 3584, intermediate 18944, vocab 152064.
QWEN7B = dict(hidden=3584, intermediate=18944, vocab=152064)

# Qwen1.5-MoE-A2.7B shapes: hidden 2048, 60 experts of intermediate 1408,
# top-4 routing, shared expert of intermediate 5632.
QWEN_MOE = dict(hidden=2048, experts=60, intermediate=1408, top_k=4, shared_intermediate=5632)


def decode_matrices_05b() -> list[MatSpec]:
    """The batch-1 decode matmul set of Qwen2.5-0.5B: per layer qkv, wo,
    gate_up (fused SwiGLU), down; then lm_head.  97 matrices, seeds 0..96 in
    this order."""
    h, i, L = QWEN05B["hidden"], QWEN05B["intermediate"], QWEN05B["layers"]
    specs = []
    seed = 0
    for layer in range(L):
        for name, M, K, sw in (("qkv", QWEN05B["qkv"], h, False), ("wo", h, h, False),
                               ("gate_up", 2 * i, h, True), ("down", h, i, False)):
            specs.append(MatSpec(f"L{layer}.{name}", M, K, sw, seed))
            seed += 1
    specs.append(MatSpec("lm_head", QWEN05B["vocab"], h, False, seed))
    return specs


def small_batch_matrices_7b() -> list[MatSpec]:
    """7B-class small-batch GEMM matrices, seeds 0, 1, 2."""
    h, i, v = QWEN7B["hidden"], QWEN7B["intermediate"], QWEN7B["vocab"]
    return [MatSpec("gate_up", 2 * i, h, True, 0), MatSpec("down", h, i, False, 1),
            MatSpec("lm_head", v, h, False, 2)]


def moe_weights(E: int = 60, H: int = 2048, I: int = 1408, I_shared: int = 5632,
                shared: bool = True):
    """MoE expert weights: expert e's gate_up [2I][H] uses seed e, its down
    [H][I] seed 1000 + e; the shared expert uses seeds E and 1000 + E.
    Returns (gate_up_all, down_all, shared_gate_up, shared_down) as GGUF bytes
    (experts concatenated in index order)."""
    gu = np.concatenate([q8_matrix(e, 2 * I, H)[0] for e in range(E)])
    dn = np.concatenate([q8_matrix(1000 + e, H, I)[0] for e in range(E)])
    if shared:
        sgu = q8_matrix(E, 2 * I_shared, H)[0]
        sdn = q8_matrix(1000 + E, H, I_shared)[0]
    else:
        sgu = sdn = None
    return gu, dn, sgu, sdn
