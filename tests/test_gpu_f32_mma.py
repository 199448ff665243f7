"""GPU parity of the tensor-core path for fp32 activations (q8_gemv_split and
q8_gate_up_swiglu_split: N >= 5, and N >= 3 for matrices with a 128-row tile
per SM or more) against the fp64 CPU oracle, through the C ABI.

That path splits each fp32 activation into three int8 terms per 32-block and
takes the block dots on tcgen05 kind::i8, so besides shapes that cover its tile
tails (128-row tiles; 64 outputs per SwiGLU tile), its K split over clusters
and K ranges that end inside a stage, these tests feed it the activation
patterns a split can get wrong: zero blocks, one large value among tiny ones,
a wide dynamic range, and exact scaling by powers of two.

Tolerance: |y - y_ref| <= 1e-5 * sum_k |w_k x_k| per element, the GEMV bar;
SwiGLU outputs carry it through silu (|silu'| <= 1.1)."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import q8gen
from q8_test_utils import TOL_REL, assert_within, matrix, pack, rows_subset, swiglu_bound
from q8_test_utils import gate_up as _gate_up
from q8_test_utils import gemv as _gemv

pytestmark = pytest.mark.gpu


def gemv(packed, x, M, K):
    return _gemv(packed, x, M, K, split=True)


def gate_up(packed, x, I, K):
    return _gate_up(packed, x, I, K, split=True)


# (M, K, N): one 128-row tile, ragged tiles, single blocks, K split over
# clusters with K ranges ending inside a stage, more tiles than SMs
GEMV_CASES = [
    (1152, 896, 5),
    (1152, 896, 8),
    (1000, 2048, 9),
    (203, 1408, 16),
    (13, 32, 16),
    (1, 64, 6),
    (300, 96, 7),      # 3 tiles, 3 blocks: one block per CTA of a cluster
    (72, 18944, 16),   # one tile, 8-CTA cluster over a long K
    (4096, 3584, 12),  # 32 tiles, K split by 4
    (20000, 256, 16),  # 157 tiles: more tiles than SMs, one stage each
    (2056, 160, 11),   # K = 5 blocks: every stage partial
    (20000, 256, 3),   # N = 3, 4 on the tensor cores: 157 tiles, one activation row per epilogue warp
    (20000, 896, 4),
    (19000, 1408, 4),  # 149 tiles, ragged last tile
]


@pytest.mark.parametrize("M,K,N", GEMV_CASES)
def test_gemv_tensor_cores_match_oracle(M, K, N):
    g, x = matrix(31 * M + K + N, M, K, N)
    y = gemv(pack(g, M, K), x, M, K)
    y_ref, y_abs = oracle.gemv(g, x, M, K, threads=oracle.max_threads())
    ratio = assert_within(y, y_ref, TOL_REL * y_abs, f"gemv M={M} K={K} N={N}")
    assert ratio < 0.5


# (I, K, N): the last tile's gate rows running past I (I not a multiple of
# 64), one packed group, clusters, many tiles
SWIGLU_CASES = [
    (200, 896, 5),
    (4864, 896, 8),
    (104, 4864, 16),
    (8, 32, 16),
    (1408, 2048, 16),
    (72, 96, 9),
    (9480, 256, 13),  # 149 tiles
    (9480, 256, 3),   # N = 3, 4 on the tensor cores (149 tiles)
    (9600, 896, 4),
]


@pytest.mark.parametrize("I,K,N", SWIGLU_CASES)
def test_swiglu_tensor_cores_match_oracle(I, K, N):
    g, x = matrix(17 * I + K + N, 2 * I, K, N)
    h = gate_up(pack(g, 2 * I, K), x, I, K)
    ref = oracle.gate_up_swiglu(g, x, I, K, threads=oracle.max_threads())
    assert_within(h, ref["h"], swiglu_bound(ref), f"swiglu I={I} K={K} N={N}")


def _edge_activations(N, K, seed):
    """Activation rows that stress the three-term split: zero blocks, a spike
    among tiny values, values spanning 1e-30..1e30 across blocks, negative
    zeros, and a row equal to another."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((N, K)).astype(np.float32)
    x[0, :32] = 0.0                                  # an all-zero block
    x[0, 32:64] = -0.0
    x[1, 64:96] = 1e-7 * rng.standard_normal(32)     # tiny values
    x[1, 70] = 3.0e4                                 # ... with one large one
    scale = np.float32(10.0) ** rng.integers(-30, 31, (K // 32,)).astype(np.float32)
    x[2] = (x[2].reshape(-1, 32) * scale[:, None]).reshape(-1)
    x[3] = np.float32(127.0)                         # amax hits 127 exactly
    x[3, 1::2] = -0.5
    x[4] = x[5 % N]                                  # duplicate rows give identical outputs
    return x


@pytest.mark.parametrize("N", [5, 8, 16])
def test_gemv_tensor_cores_edge_activations(N):
    M, K = 520, 1024
    g, _ = matrix(909, M, K)
    x = _edge_activations(N, K, 910 + N)
    y = gemv(pack(g, M, K), x, M, K)
    y_ref, y_abs = oracle.gemv(g, x, M, K, threads=oracle.max_threads())
    assert_within(y, y_ref, TOL_REL * y_abs, f"edge activations N={N}")
    assert np.array_equal(y[4], y[5 % N])


def test_gemv_tensor_cores_exact_scaling():
    """Scaling every d by 2, or x by 2, doubles y bit for bit (the split of x is
    scale-invariant under powers of two, and d_w multiplies an exact sum)."""
    M, K, N = 700, 1408, 8
    g, x = matrix(77, M, K, N)
    q, dbits = q8gen.split_gguf(g, M, K)
    d2 = (dbits.view(np.float16).astype(np.float32) * 2).astype(np.float16).view(np.uint16)
    p = pack(g, M, K)
    y1 = gemv(p, x, M, K)
    assert np.array_equal(gemv(pack(q8gen.assemble_gguf(q, d2), M, K), x, M, K), 2 * y1)
    assert np.array_equal(gemv(p, 2 * x, M, K), 2 * y1)
    assert np.array_equal(gemv(p, -x, M, K), -y1)


def test_gemv_tensor_cores_one_hot_is_exact():
    """Unit scales and one-hot rows of x return columns of q exactly."""
    M, K, N = 260, 96, 8
    rng = np.random.default_rng(4)
    q = rng.integers(-127, 128, (M, K), dtype=np.int8)
    g = q8gen.assemble_gguf(q, np.full((M, K // 32), 0x3C00, np.uint16))
    ks = [0, 5, 31, 32, 47, 63, 64, 95]
    x = np.zeros((N, K), np.float32)
    for n, k in enumerate(ks):
        x[n, k] = 1.0
    y = gemv(pack(g, M, K), x, M, K)
    for n, k in enumerate(ks):
        assert np.array_equal(y[n], q[:, k].astype(np.float32))


def test_gemv_tensor_cores_deterministic():
    M, K, N = 3000, 4864, 16  # 24 tiles: K split over 6-CTA clusters
    g, x = matrix(12, M, K, N)
    p = pack(g, M, K)
    assert np.array_equal(gemv(p, x, M, K), gemv(p, x, M, K))


@pytest.mark.parametrize("M,K", [(152064, 3584), (3584, 18944)])
@pytest.mark.parametrize("N", [8, 16])
def test_gemv_tensor_cores_full_size_sampled(M, K, N):
    """7B-class lm_head / down at N = 8, 16 (the small-batch workload), sampled
    rows checked against the oracle row by row."""
    g, x = matrix(5150 + M + N, M, K, N)
    y = gemv(pack(g, M, K), x, M, K)
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([np.arange(8), np.arange(M - 8, M), rng.integers(0, M, 160),
                                     np.arange(127, M, 8192)]))
    y_ref, y_abs = oracle.gemv(rows_subset(g, M, K, rows), x, len(rows), K, threads=oracle.max_threads())
    assert_within(y[:, rows], y_ref, TOL_REL * y_abs, f"full-size {M}x{K} N={N}")


@pytest.mark.parametrize("N", [8, 16])
def test_swiglu_tensor_cores_full_size_sampled(N):
    """7B-class gate_up (37888 x 3584) at N = 8, 16, sampled outputs."""
    I, K = 18944, 3584
    g, x = matrix(4343 + N, 2 * I, K, N)
    h = gate_up(pack(g, 2 * I, K), x, I, K)
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([np.arange(8), np.arange(I - 8, I), rng.integers(0, I, 120),
                                     np.arange(63, I, 4096)]))
    sub = np.concatenate([rows_subset(g, 2 * I, K, rows), rows_subset(g, 2 * I, K, rows + I)])
    ref = oracle.gate_up_swiglu(sub, x, len(rows), K, threads=oracle.max_threads())
    assert_within(h[:, rows], ref["h"], swiglu_bound(ref), f"gate_up full size N={N}")


def _spike_case(M, K, N, seed):
    """A crafted input the split cannot represent to the GEMV bar: in every
    32-block of x one value 1e6 times the others, and in every weight row
    q = 0 exactly where that value sits, so sum_k |w_k x_k| sees only the small
    values while the split's residual scales with the large one."""
    rng = np.random.default_rng(seed)
    q = rng.integers(-127, 128, (M, K), dtype=np.int8)
    q[q == 0] = 1
    d = (np.abs(rng.standard_normal((M, K // 32))) * 0.02).astype(np.float16).view(np.uint16)
    x = (rng.standard_normal((N, K)) * 1e-3).astype(np.float32)
    spike = rng.integers(0, 32, K // 32)
    for b, i in enumerate(spike):
        x[:, 32 * b + i] = 1e3
        q[:, 32 * b + i] = 0
    return q8gen.assemble_gguf(q, d), x


def test_spike_on_zero_weight_default_path_keeps_the_bar():
    """The default entry point (CUDA cores) meets 1e-5 * sum|w x| on the
    crafted input; the split entry point stays within its own documented
    bound there, 1e-5 * sum|w x| + 2.5e-7 * sum_b amax_b * sum_{k in b} |w_k|."""
    M, K, N = 2048, 896, 8
    g, x = _spike_case(M, K, N, 91)
    p = pack(g, M, K)
    y_ref, y_abs = oracle.gemv(g, x, M, K, threads=oracle.max_threads())
    y_def = _gemv(p, x, M, K)
    assert_within(y_def, y_ref, TOL_REL * y_abs, "default path, spike on zero weight")
    y_split = gemv(p, x, M, K)
    qw, dbits = q8gen.split_gguf(g, M, K)
    wabs = np.abs(qw.astype(np.float64) * np.repeat(dbits.view(np.float16).astype(np.float64), 32, axis=1))
    amax = np.abs(x.astype(np.float64)).reshape(N, K // 32, 32).max(axis=2)            # [N][B]
    wsum = wabs.reshape(M, K // 32, 32).sum(axis=2)                                  # [M][B]
    split_bound = TOL_REL * y_abs + 2.5e-7 * (amax @ wsum.T)
    assert_within(y_split, y_ref, split_bound, "split path within its stated bound")
