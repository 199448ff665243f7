"""GPU parity of the integer path (S7 activation quantisation, S8 Q8 x Q8
block dots and product) and the MoE router (S5) against the CPU oracle.

Bars: quantised activations (q bytes and binary16 scale bits) and int32 block
dots are bit-exact; Q8 x Q8 outputs are within 1e-5 * sum_b |d_w d_x| sum_i |q_w q_x|;
router indices are exact and weights within 1e-6 relative (fp32 softmax
against the fp64 oracle)."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import q8gen
from q8_test_utils import TOL_REL, assert_within, dev, pack, rows_subset, torch

pytestmark = pytest.mark.gpu


def q8():
    import q8_block_quantized_02_b200 as m
    return m


def gpu_quantize(x: np.ndarray):
    t = torch()
    N, K = x.shape
    xq = t.empty((N, K), dtype=t.int8, device="cuda")
    xd = t.empty((N, K // 32), dtype=t.int16, device="cuda")
    q8().q8_quantize_act(dev(x.astype(np.float32)), xq, xd, N, K)
    return xq.cpu().numpy(), xd.cpu().numpy().view(np.uint16)


# --------------------------------------------------------------------------
# S7 activation quantisation: bit-exact
# --------------------------------------------------------------------------

@pytest.mark.parametrize("N,K", [(1, 896), (16, 3584), (1, 4864), (16, 18944), (3, 32), (5, 96)])
def test_quantize_act_bit_exact(N, K):
    x = q8gen.activations(N * 1000 + K, N, K)
    q, d = gpu_quantize(x)
    q_ref, d_ref, _ = oracle.quantize_act(x)
    assert np.array_equal(q, q_ref)
    assert np.array_equal(d, d_ref)


def test_quantize_act_edge_values():
    rng = np.random.default_rng(4)
    K = 32 * 12
    x = (rng.standard_normal((4, K)) * np.exp(rng.uniform(-40, 40, (4, K // 32)).repeat(32, axis=1))).astype(np.float32)
    x[0, :32] = 0.0                                 # all-zero block
    x[0, 32:64] = np.float32(1e-40)                 # subnormal inputs
    x[1, :32] = [127, 0.5, -0.5, 1.5, 2.5, -63.5, 126.5] + [0] * 25  # half-away ties
    x[2, :32] = -np.float32(3.0e38)                 # huge, d overflows binary16
    x[3, 64:96] = np.linspace(-1, 1, 32, dtype=np.float32)
    q, d = gpu_quantize(x)
    with np.errstate(over="ignore"):
        q_ref, d_ref, _ = oracle.quantize_act(x)
    assert np.array_equal(q, q_ref)
    assert np.array_equal(d, d_ref)
    assert q[1, :7].tolist() == [127, 1, -1, 2, 3, -64, 127]


# --------------------------------------------------------------------------
# S8 block dots: bit-exact; Q8 x Q8 product within tolerance
# --------------------------------------------------------------------------

@pytest.mark.parametrize("M,K,N", [(4096, 896, 1), (4096, 896, 16), (203, 3584, 3), (13, 32, 2)])
def test_block_dots_bit_exact(M, K, N):
    g, x = q8gen.q8_matrix(M + K + N, M, K, N)
    xq, xd, _ = oracle.quantize_act(x)
    t = torch()
    dots = t.empty((N, M, K // 32), dtype=t.int32, device="cuda")
    q8().q8q8_block_dots(pack(g, M, K), dev(xq), dots, M, K, N)
    ref, _, _ = oracle.q8q8(g, xq, xd, M, K, threads=oracle.max_threads())
    assert np.array_equal(dots.cpu().numpy(), ref)


def run_q8q8(g, xq, xd, M, K):
    t = torch()
    N = xq.shape[0]
    y = t.full((N, M), float("nan"), dtype=t.float32, device="cuda")
    q8().q8q8_gemv(pack(g, M, K), dev(xq), dev(xd.view(np.int16)), y, M, K, N)
    return y.cpu().numpy()


@pytest.mark.parametrize("K", [896, 3584, 4864, 18944])
@pytest.mark.parametrize("N", [1, 16])
def test_q8q8_gemv_matches_oracle(K, N):
    """The Q8 x Q8 sweep: M = 4096, K in {896, 3584, 4864, 18944}, N in {1, 16}."""
    M = 4096
    g, x = q8gen.q8_matrix(K * 3 + N, M, K, N)
    xq, xd, _ = oracle.quantize_act(x)
    y = run_q8q8(g, xq, xd, M, K)
    rows = np.arange(M) if K * N <= 3584 * 16 else np.unique(np.random.default_rng(K).integers(0, M, 512))
    _, y_ref, y_abs = oracle.q8q8(rows_subset(g, M, K, rows), xq, xd, len(rows), K, want_dots=False,
                                  threads=oracle.max_threads())
    assert_within(y[:, rows], y_ref, TOL_REL * y_abs, f"q8q8 K={K} N={N}")


@pytest.mark.parametrize("M,K,N", [(13, 32, 1), (203, 1408, 2), (1000, 2048, 4), (72, 18944, 8), (8, 64, 16)])
def test_q8q8_ragged_shapes(M, K, N):
    g, x = q8gen.q8_matrix(M * 5 + K + N, M, K, N)
    xq, xd, _ = oracle.quantize_act(x)
    y = run_q8q8(g, xq, xd, M, K)
    _, y_ref, y_abs = oracle.q8q8(g, xq, xd, M, K, want_dots=False)
    assert_within(y, y_ref, TOL_REL * y_abs, f"q8q8 {M}x{K} N={N}")


@pytest.mark.parametrize("M,K,N", [
    (4096, 896, 9),        # K split over a cluster of 4, one stage per CTA
    (4096, 3584, 12),      # cluster of 4, pipelined stages
    (1000, 2048, 13),      # ragged last tile (125 groups)
    (136, 96, 16),         # 17 groups: a tile of 16 and a tile of 1; 3 blocks over 3 CTAs
    (896, 896, 16),        # cluster of 8, 3-4 blocks per CTA (partial stage)
    (3584, 18944, 16),     # cluster of 5 with uneven K slices
    (37888, 3584, 16),     # one CTA per SM walking two tiles
    (151936, 896, 16),     # 1187 tiles: the vocabulary projection
])
def test_q8q8_tensor_core_shapes(M, K, N):
    """N >= 9 runs on the tcgen05 kernel: 128-row tiles, K split across a
    cluster when there are fewer tiles than SMs."""
    g, x = q8gen.q8_matrix(M + 7 * K + N, M, K, N)
    xq, xd, _ = oracle.quantize_act(x)
    y = run_q8q8(g, xq, xd, M, K)
    assert np.all(np.isfinite(y))
    if M * K <= 4096 * 3584:
        rows = np.arange(M)
    else:
        rng = np.random.default_rng(M + K)
        rows = np.unique(np.concatenate([rng.integers(0, M, 384), np.arange(128), np.arange(M - 136, M)]))
    _, y_ref, y_abs = oracle.q8q8(rows_subset(g, M, K, rows), xq, xd, len(rows), K, want_dots=False,
                                  threads=oracle.max_threads())
    assert_within(y[:, rows], y_ref, TOL_REL * y_abs, f"q8q8 tensor cores {M}x{K} N={N}")


def test_q8q8_tensor_core_deterministic_and_exact_on_integers():
    """Run-to-run identical; with unit scales every output is an exact integer
    sum of block dots, so the result must equal the oracle's exactly."""
    M, K, N = 4096, 3584, 16
    g, x = q8gen.q8_matrix(5, M, K, N)
    xq, xd, _ = oracle.quantize_act(x)
    y1 = run_q8q8(g, xq, xd, M, K)
    y2 = run_q8q8(g, xq, xd, M, K)
    assert np.array_equal(y1, y2)
    # scales of exactly 1.0 (binary16 0x3C00): y = sum of int32 block dots,
    # which fp32 holds exactly while |partial sums| < 2^24
    qw, _ = q8gen.split_gguf(g, M, K)
    g1 = q8gen.assemble_gguf(qw, np.full((M, K // 32), 0x3C00, np.uint16))
    xd1 = np.full_like(xd, 0x3C00)
    y = run_q8q8(g1, xq, xd1, M, K)
    dots, y_ref, _ = oracle.q8q8(g1, xq, xd1, M, K, threads=oracle.max_threads())
    assert np.array_equal(y.astype(np.float64), y_ref)


@pytest.mark.parametrize("M,K,N", [
    (4096, 896, 1),      # 8-consumer-warp column kernel
    (4096, 18944, 1),    # 16-warp kernel (a CTA's share of the weights >= 256 KB)
    (37888, 3584, 1),    # 16-warp kernel, 32 row groups per CTA, two consumer groups
    (4096, 896, 2),
    (4096, 18944, 2),
    (1000, 3584, 3),     # N = 3 on the 4-column build, ragged last group
    (4096, 18944, 4),
    (37888, 3584, 4),
])
def test_q8q8_cuda_cores_exact_on_integers(M, K, N):
    """The dp4a kernels (N <= 4): with unit scales every output is the exact
    integer sum of the int32 block dots (int8 x int8 accumulated exactly, the
    scales applied per block -- the GPULlama3.java Qwen1.5-MoE pull request,
    "Key implementation notes"), which fp32 holds exactly while partial sums
    stay below 2^24; so y must equal the oracle's sum of block dots bit for
    bit, at the shapes that take the 8- and 16-warp column kernels."""
    g, x = q8gen.q8_matrix(M + 3 * K + N, M, K, N)
    xq, _, _ = oracle.quantize_act(x)
    qw, _ = q8gen.split_gguf(g, M, K)
    g1 = q8gen.assemble_gguf(qw, np.full((M, K // 32), 0x3C00, np.uint16))
    xd1 = np.full((N, K // 32), 0x3C00, np.uint16)
    y = run_q8q8(g1, xq, xd1, M, K)
    dots, y_ref, _ = oracle.q8q8(g1, xq, xd1, M, K, threads=oracle.max_threads())
    assert np.abs(y_ref).max() < 2 ** 24
    assert np.array_equal(dots.sum(axis=2, dtype=np.int64).astype(np.float64), y_ref)
    assert np.array_equal(y.astype(np.float64), y_ref)


def test_quantize_then_q8q8_end_to_end():
    """GPU quantiser feeding the GPU product equals the oracle chain."""
    M, K, N = 4096, 3584, 16
    g, x = q8gen.q8_matrix(77, M, K, N)
    t = torch()
    xq = t.empty((N, K), dtype=t.int8, device="cuda")
    xd = t.empty((N, K // 32), dtype=t.int16, device="cuda")
    y = t.empty((N, M), dtype=t.float32, device="cuda")
    q8().q8_quantize_act(dev(x), xq, xd, N, K)
    q8().q8q8_gemv(pack(g, M, K), xq, xd, y, M, K, N)
    q_ref, d_ref, _ = oracle.quantize_act(x)
    assert np.array_equal(xq.cpu().numpy(), q_ref)
    _, y_ref, y_abs = oracle.q8q8(g, q_ref, d_ref, M, K, want_dots=False, threads=oracle.max_threads())
    assert_within(y.cpu().numpy(), y_ref, TOL_REL * y_abs, "quantize -> q8q8")


# --------------------------------------------------------------------------
# S5 router
# --------------------------------------------------------------------------

def gpu_route(logits: np.ndarray, k: int, renorm: bool = False):
    t = torch()
    T, E = logits.shape
    idx = t.empty((T, k), dtype=t.int32, device="cuda")
    w = t.empty((T, k), dtype=t.float32, device="cuda")
    q8().q8_moe_route(dev(logits), T, E, k, renorm, idx, w)
    return idx.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("T", [1, 8, 16])
@pytest.mark.parametrize("renorm", [False, True])
def test_route_matches_oracle(T, renorm):
    lg = q8gen.logits(T + 61, T, 60)
    idx, w = gpu_route(lg, 4, renorm)
    idx_ref, w_ref = oracle.route(lg, 4, renorm)
    assert np.array_equal(idx, idx_ref)
    assert np.all(np.abs(w - w_ref) <= 1e-6 * w_ref)


def test_route_ties_and_limits():
    E = 60
    lg = np.full((3, E), -2.0, np.float32)
    lg[0, [7, 3, 40, 12, 5]] = 1.0           # five-way tie for four slots
    lg[1] = 0.0                                # all equal
    lg[2] = np.arange(E, dtype=np.float32)     # ramp
    idx, w = gpu_route(lg, 4)
    assert idx.tolist() == [[3, 5, 7, 12], [0, 1, 2, 3], [59, 58, 57, 56]]
    idx_ref, w_ref = oracle.route(lg, 4)
    assert np.array_equal(idx, idx_ref)
    assert np.all(np.abs(w - w_ref) <= 1e-6 * w_ref)
    # the largest supported expert count and top-k
    lg2 = q8gen.logits(5, 2, 256)
    idx2, w2 = gpu_route(lg2, 8)
    idx2_ref, w2_ref = oracle.route(lg2, 8)
    assert np.array_equal(idx2, idx2_ref)
    assert np.all(np.abs(w2 - w2_ref) <= 1e-6 * w2_ref)


def test_route_rejects_bad_sizes():
    m = q8()
    t = torch()
    lg = dev(np.zeros((2, 60), np.float32))
    idx = t.empty((2, 4), dtype=t.int32, device="cuda")
    w = t.empty((2, 4), dtype=t.float32, device="cuda")
    for args, want in (((lg, 2, 60, 61, 0, idx, w), 2), ((lg, 17, 60, 4, 0, idx, w), 5),
                       ((lg, 2, 300, 4, 0, idx, w), 5), ((lg, 2, 60, 4, 2, idx, w), 1)):
        with pytest.raises(m.Q8Error) as e:
            m.q8_moe_route(*args)
        assert e.value.status == want
