"""GPU parity of the packer (S1), the fp32 GEMV/GEMM (S2/S3) and the fused
gate_up + SwiGLU (S4) against the fp64 CPU oracle, through the C ABI.

Tolerance: |y - y_ref| <= 1e-5 * sum_k |w_k x_k| for every element (GEMV and
GEMM); SwiGLU outputs carry that error through silu (|silu'| <= 1.1)."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import q8gen
from q8_test_utils import (TOL_REL, assert_within, dev, dev_bytes, gate_up, gemv, matrix, pack,
                           rows_subset, swiglu_bound, torch)

pytestmark = pytest.mark.gpu


def q8():
    import q8_block_quantized_02_b200 as m
    return m


# --------------------------------------------------------------------------
# S1 packer
# --------------------------------------------------------------------------

@pytest.mark.parametrize("M,K", [(1, 32), (7, 64), (8, 896), (13, 96), (1152, 896), (33, 4864)])
def test_pack_round_trip_bit_exact(M, K):
    g, _ = matrix(100 + M, M, K)
    t = torch()
    packed = pack(g, M, K)
    assert packed.numel() == q8().q8_packed_bytes(M, K)
    back = t.zeros(g.size, dtype=t.uint8, device="cuda")
    q8().q8_unpack_weights(packed, M, K, back)
    assert np.array_equal(back.cpu().numpy(), g)


def test_pack_layout_matches_header():
    """Spot-check the documented packed layout byte by byte."""
    M, K = 11, 64
    g, _ = matrix(5, M, K)
    p = pack(g, M, K).cpu().numpy()
    q, dbits = q8gen.split_gguf(g, M, K)
    B = K // 32
    for row in range(16):
        grp, r = divmod(row, 8)
        base = grp * 272 * B
        for c in range(2 * B):
            piece = p[base + c * 128 + r * 16: base + c * 128 + r * 16 + 16]
            want = (q[row, 16 * c:16 * c + 16].view(np.uint8) ^ 0x80) if row < M else np.full(16, 0x80, np.uint8)
            assert np.array_equal(piece, want)
        for b in range(B):
            dpos = base + 256 * B + b * 16 + r * 2
            got = int(p[dpos]) | (int(p[dpos + 1]) << 8)
            assert got == (int(dbits[row, b]) if row < M else 0)


# --------------------------------------------------------------------------
# S2 / S3 GEMV and small-batch GEMM
# --------------------------------------------------------------------------

SHAPES = [
    (1152, 896),   # Qwen2.5-0.5B fused qkv (the single-GEMV workload)
    (896, 4864),   # down projection shape (long K)
    (13, 32),      # one block, ragged rows
    (1, 64),       # a single row
    (203, 1408),   # ragged rows, MoE expert K
    (1000, 2048),  # several tiles, K not a power-of-two multiple of a stage
    (72, 18944),   # very long K (7B-class down)
]


# every shape at every N (N >= 5: the group-owner kernel on the CUDA cores)
GEMV_CASES = [(M, K, N) for N in (1, 2, 3, 4, 5, 8, 16) for (M, K) in SHAPES]


@pytest.mark.parametrize("M,K,N", GEMV_CASES)
def test_gemv_matches_oracle(M, K, N):
    g, x = matrix(M * 7 + K + N, M, K, N)
    y = gemv(pack(g, M, K), x, M, K)
    y_ref, y_abs = oracle.gemv(g, x, M, K, threads=oracle.max_threads())
    assert_within(y, y_ref, TOL_REL * y_abs, f"gemv M={M} K={K} N={N}")


def test_gemv_config0_exact_seed():
    """The single-GEMV workload exactly as specified: 1152 x 896, N = 1, seed 0."""
    g, x = q8gen.q8_matrix(0, 1152, 896, 1)
    y = gemv(pack(g, 1152, 896), x, 1152, 896)
    y_ref, y_abs = oracle.gemv(g, x, 1152, 896)
    ratio = assert_within(y, y_ref, TOL_REL * y_abs, "config0")
    assert ratio < 0.1  # fp32 error is far inside the stated tolerance


def test_gemv_one_hot_is_exact():
    """Unit scales and one-hot x return a column of q exactly (closed form)."""
    M, K = 40, 96
    rng = np.random.default_rng(3)
    q = rng.integers(-127, 128, (M, K), dtype=np.int8)
    g = q8gen.assemble_gguf(q, np.full((M, K // 32), 0x3C00, np.uint16))
    p = pack(g, M, K)
    for k in (0, 17, 32, 95):
        x = np.zeros((1, K), np.float32)
        x[0, k] = 1.0
        assert np.array_equal(gemv(p, x, M, K)[0], q[:, k].astype(np.float32))


def test_gemv_linear_in_d_exactly():
    M, K = 300, 896
    g, x = matrix(77, M, K, 2)
    q, dbits = q8gen.split_gguf(g, M, K)
    d2 = (dbits.view(np.float16).astype(np.float32) * 2).astype(np.float16).view(np.uint16)
    y1 = gemv(pack(g, M, K), x, M, K)
    y2 = gemv(pack(q8gen.assemble_gguf(q, d2), M, K), x, M, K)
    assert np.array_equal(y2, 2 * y1)
    y3 = gemv(pack(g, M, K), 2 * x, M, K)
    assert np.array_equal(y3, 2 * y1)


def test_gemv_zero_rows_are_zero():
    M, K = 24, 64
    g, x = matrix(8, M, K, 3)
    q, dbits = q8gen.split_gguf(g, M, K)
    q[5] = 0
    dbits[9] = 0
    y = gemv(pack(q8gen.assemble_gguf(q, dbits), M, K), x, M, K)
    assert np.all(y[:, 5] == 0) and np.all(y[:, 9] == 0)


def test_gemv_deterministic():
    M, K = 5000, 896
    g, x = matrix(9, M, K, 1)
    p = pack(g, M, K)
    a = gemv(p, x, M, K)
    b = gemv(p, x, M, K)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("M,K", [(151936, 896), (152064, 3584), (3584, 18944)])
def test_gemv_full_size_sampled(M, K):
    """Full-size lm_head / down matrices at the bench's launch shape; a sample of
    rows (first, last, every tile boundary region, random) checked against the
    oracle row by row."""
    g, x = matrix(2024 + M, M, K, 1)
    y = gemv(pack(g, M, K), x, M, K)
    rng = np.random.default_rng(1)
    rows = np.unique(np.concatenate([np.arange(16), np.arange(M - 16, M), rng.integers(0, M, 400),
                                     np.arange(127, M, 4096)]))
    sub = rows_subset(g, M, K, rows)
    y_ref, y_abs = oracle.gemv(sub, x, len(rows), K, threads=oracle.max_threads())
    assert_within(y[:, rows], y_ref, TOL_REL * y_abs, f"full-size {M}x{K}")


@pytest.mark.parametrize("M,K", [(152064, 3584), (3584, 18944)])
@pytest.mark.parametrize("N", [2, 4, 8, 16])
def test_gemv_full_size_sampled_small_batch(M, K, N):
    """The 7B-class lm_head and down at N = 2, 4, 8 and 16 (the small-batch
    sweep), full size, at the launch shape the planner picks for them on the
    CUDA cores; sampled rows against the oracle."""
    g, x = matrix(3030 + M + N, M, K, N)
    y = gemv(pack(g, M, K), x, M, K)
    rng = np.random.default_rng(N)
    rows = np.unique(np.concatenate([np.arange(16), np.arange(M - 16, M), rng.integers(0, M, 300),
                                     np.arange(127, M, 4096)]))
    y_ref, y_abs = oracle.gemv(rows_subset(g, M, K, rows), x, len(rows), K, threads=oracle.max_threads())
    assert_within(y[:, rows], y_ref, TOL_REL * y_abs, f"full-size {M}x{K} N={N}")


# --------------------------------------------------------------------------
# S4 fused gate_up + SwiGLU
# --------------------------------------------------------------------------

SWIGLU_SHAPES = [(4864, 896), (8, 32), (1408, 2048), (104, 4864), (200, 896)]
SWIGLU_CASES = [(I, K, N) for N in (1, 2, 5, 8, 16) for (I, K) in SWIGLU_SHAPES]


@pytest.mark.parametrize("I,K,N", SWIGLU_CASES)
def test_gate_up_swiglu_matches_oracle(I, K, N):
    g, x = matrix(I + K + N, 2 * I, K, N)
    h = gate_up(pack(g, 2 * I, K), x, I, K)
    ref = oracle.gate_up_swiglu(g, x, I, K, threads=oracle.max_threads())
    assert_within(h, ref["h"], swiglu_bound(ref), f"swiglu I={I} K={K} N={N}")


@pytest.mark.parametrize("N", [1, 2, 4, 8, 16])
def test_gate_up_full_size_sampled(N):
    """7B-class gate_up (37888 x 3584) at N = 1, 2, 4, 8 and 16, sampled rows."""
    I, K = 18944, 3584
    g, x = matrix(4242 + (N - 1) * 7, 2 * I, K, N)
    h = gate_up(pack(g, 2 * I, K), x, I, K)
    rng = np.random.default_rng(2 + N)
    rows = np.unique(np.concatenate([np.arange(8), np.arange(I - 8, I), rng.integers(0, I, 300)]))
    sub = np.concatenate([rows_subset(g, 2 * I, K, rows), rows_subset(g, 2 * I, K, rows + I)])
    ref = oracle.gate_up_swiglu(sub, x, len(rows), K, threads=oracle.max_threads())
    assert_within(h[:, rows], ref["h"], swiglu_bound(ref), "gate_up full size")


# --------------------------------------------------------------------------
# argument validation (host side; nothing is launched)
# --------------------------------------------------------------------------

def test_validation_rejects_bad_arguments():
    m = q8()
    t = torch()
    M, K = 16, 64
    g, x = matrix(1, M, K, 1)
    p = pack(g, M, K)
    xd = dev(x)
    y = t.empty((1, M), dtype=t.float32, device="cuda")
    host = t.empty((1, M), dtype=t.float32)

    def status(fn, *a):
        with pytest.raises(m.Q8Error) as e:
            fn(*a)
        return e.value.status

    assert status(m.q8_gemv, p, xd, y, M, 48, 1) == 2          # K % 32
    assert status(m.q8_gemv, p, xd, y, 0, K, 1) == 2           # M <= 0
    assert status(m.q8_gemv, p, xd, y, M, K, 17) == 5          # N > 16
    assert status(m.q8_gemv, p, xd, host, M, K, 1) == 4        # host output
    assert status(m.q8_gemv, 0, xd, y, M, K, 1) == 1           # null
    assert status(m.q8_gemv, p.data_ptr() + 4, xd, y, M, K, 1) == 3  # misaligned
    assert status(m.q8_gate_up_swiglu, p, xd, y, 4, K, 1) == 2  # I % 8
    assert m.q8_read_device_error() == (0, 0)


def test_cuda_graph_replay_matches_eager():
    m = q8()
    t = torch()
    M, K = 9728, 896
    g, x = matrix(55, M, K, 1)
    p = pack(g, M, K)
    xd = dev(x)
    y = t.empty((1, M // 2), dtype=t.float32, device="cuda")
    m.q8_gate_up_swiglu(p, xd, y, M // 2, K, 1)
    eager = y.clone()
    s = t.cuda.Stream()
    graph = t.cuda.CUDAGraph()
    with t.cuda.stream(s):
        m.q8_gate_up_swiglu(p, xd, y, M // 2, K, 1, stream=s)  # warm on the side stream
        s.synchronize()
        with t.cuda.graph(graph, stream=s):
            m.q8_gate_up_swiglu(p, xd, y, M // 2, K, 1, stream=s)
    y.zero_()
    graph.replay()
    t.cuda.synchronize()
    assert t.equal(y, eager)
