"""GPU parity of the K-quant GEMV (q8_q4k_gemv, q8_q6k_gemv: GGUF Q4_K / Q6_K
super-blocks read in their raw layout; q8_q6k_gemv_packed from the re-laid
Q6_K units, with the pack layout and round trip) against the fp64 CPU oracle,
through the C ABI.  Every packed field is random bytes, so all scale/min bit
patterns and all nibble values occur.

Tolerance: |y - y_ref| <= 1e-5 * sum_k |w_k x_k| per element, the GEMV bar."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import q8gen
from q8_test_utils import TOL_REL, assert_within, dev, pack_q6k_reference, torch

pytestmark = pytest.mark.gpu

BYTES = {"q4_k": 144, "q6_k": 210}


def q8():
    import q8_block_quantized_02_b200 as m
    return m


def run(fmt, blocks, x, M, K):
    t = torch()
    N = x.shape[0]
    w = t.from_numpy(blocks.copy()).cuda()
    y = t.full((N, M), float("nan"), dtype=t.float32, device="cuda")
    fn = q8().q8_q4k_gemv if fmt == "q4_k" else q8().q8_q6k_gemv
    fn(w, dev(x), y, M, K, N)
    return y.cpu().numpy()


@pytest.mark.parametrize("fmt", ["q4_k", "q6_k"])
@pytest.mark.parametrize("M,K,N", [(1, 256, 1), (13, 512, 2), (1000, 3584, 4), (37, 2048, 3),
                                   (3584, 18944, 1), (4096, 3584, 2),
                                   # Q4_K runs the tile kernel: tiles of 32 rows (ragged
                                   # last tile), blocks split over 8 warps; SB = 1 leaves
                                   # seven warps without a block
                                   (33, 256, 1), (4739, 2304, 1), (70, 4864, 2), (5000, 1024, 2)])
def test_kquant_gemv_matches_oracle(fmt, M, K, N):
    blocks = q8gen.kquant_matrix(fmt, 5 * M + K + N, M, K)
    x = q8gen.activations(M + 2 * K + N, N, K)
    y = run(fmt, blocks, x, M, K)
    y_ref, y_abs = oracle.kquant_gemv(fmt, blocks, x, M, K, threads=oracle.max_threads())
    assert_within(y, y_ref, TOL_REL * y_abs, f"{fmt} M={M} K={K} N={N}")


@pytest.mark.parametrize("fmt", ["q4_k", "q6_k"])
def test_kquant_full_size_sampled(fmt):
    """7B-class lm_head shape 152064 x 3584 at N = 1, sampled rows (rows are
    contiguous runs of blocks, so a row subset is a slice of the bytes)."""
    M, K, N = 152064, 3584, 1
    blocks = q8gen.kquant_matrix(fmt, 777, M, K)
    x = q8gen.activations(778, N, K)
    y = run(fmt, blocks, x, M, K)
    rows = np.unique(np.concatenate([np.arange(4), np.arange(M - 4, M),
                                     np.random.default_rng(0).integers(0, M, 200)]))
    per_row = (K // 256) * BYTES[fmt]
    sub = blocks.reshape(M, per_row)[rows].reshape(-1)
    y_ref, y_abs = oracle.kquant_gemv(fmt, sub, x, len(rows), K, threads=oracle.max_threads())
    assert_within(y[:, rows], y_ref, TOL_REL * y_abs, f"{fmt} full size")


def test_kquant_deterministic_and_rejections():
    t = torch()
    M, K = 500, 1024
    blocks = q8gen.kquant_matrix("q4_k", 3, M, K)
    x = q8gen.activations(4, 2, K)
    assert np.array_equal(run("q4_k", blocks, x, M, K), run("q4_k", blocks, x, M, K))
    w = t.from_numpy(blocks.copy()).cuda()
    y = t.empty((5, M), dtype=t.float32, device="cuda")
    with pytest.raises(q8().Q8Error) as e:
        q8().q8_q4k_gemv(w, dev(np.zeros((1, 992), np.float32)), y, M, 992, 1)  # K % 256 != 0
    assert e.value.status == 2
    with pytest.raises(q8().Q8Error) as e:
        q8().q8_q6k_gemv(w, dev(np.zeros((5, K), np.float32)), y, M, K, 5)    # N > 4
    assert e.value.status == 5


@pytest.mark.parametrize("N", [1, 2, 4])
def test_q4k_zero_weight_sub_blocks(N):
    """Sub-blocks whose weights are all exactly zero (every nibble q with
    d*sc*q = dmin*m) contribute nothing: sum |w x| then sees only the other
    sub-blocks, so a kernel whose rounding scaled with d*sc*sum(q x) or
    dmin*m*sum(x) instead of with each weight would miss the bar here."""
    M, K = 300, 1024
    rng = np.random.default_rng(17)
    blocks = q8gen.kquant_matrix("q4_k", 19, M, K).reshape(M, K // 256, 144).copy()
    # d = dmin = 1.0 (binary16 0x3C00); sub-block 0: scale 4, min 12 and every
    # nibble 3, so w = 4 * 3 - 12 = 0 exactly; sub-blocks 1-7 keep random codes
    blocks[:, :, 0:2] = np.frombuffer(np.uint16(0x3C00).tobytes(), np.uint8)
    blocks[:, :, 2:4] = np.frombuffer(np.uint16(0x3C00).tobytes(), np.uint8)
    blocks[:, :, 4] = (blocks[:, :, 4] & 0xC0) | 4          # sc of sub-block 0
    blocks[:, :, 8] = (blocks[:, :, 8] & 0xC0) | 12         # m of sub-block 0
    blocks[:, :, 16:48] = (blocks[:, :, 16:48] & 0xF0) | 3  # low nibbles of bytes 0..31: sub-block 0
    x = (rng.standard_normal((N, K)) * 10).astype(np.float32)
    flat = blocks.reshape(-1)
    y = run("q4_k", flat, x, M, K)
    y_ref, y_abs = oracle.kquant_gemv("q4_k", flat, x, M, K, threads=oracle.max_threads())
    assert_within(y, y_ref, TOL_REL * y_abs, f"q4_k zero-weight sub-blocks N={N}")


# ---------------------------------------------------------------------------
# Q6_K packed units (q8_q6k_pack_weights / q8_q6k_gemv_packed)
# ---------------------------------------------------------------------------
def pack_q6k(blocks, M, K):
    t = torch()
    raw = t.from_numpy(blocks.copy()).cuda()
    packed = t.full((q8().q8_q6k_packed_bytes(M, K),), 0xA5, dtype=t.uint8, device="cuda")
    q8().q8_q6k_pack_weights(raw, M, K, packed)
    return packed


def run_q6k_packed(packed, x, M, K):
    t = torch()
    N = x.shape[0]
    y = t.full((N, M), float("nan"), dtype=t.float32, device="cuda")
    q8().q8_q6k_gemv_packed(packed, dev(x), y, M, K, N)
    return y.cpu().numpy()


@pytest.mark.parametrize("M,K", [(1, 256), (45, 512), (100, 3584), (64, 18944)])
def test_q6k_pack_layout_and_round_trip(M, K):
    t = torch()
    blocks = q8gen.kquant_matrix("q6_k", 91 + M, M, K)
    packed = pack_q6k(blocks, M, K)
    assert packed.numel() == -(-M // 32) * (K // 256) * 6720
    assert np.array_equal(packed.cpu().numpy(), pack_q6k_reference(blocks, M, K))
    raw = t.full((blocks.size,), 0x5A, dtype=t.uint8, device="cuda")
    q8().q8_q6k_unpack_weights(packed, M, K, raw)
    assert np.array_equal(raw.cpu().numpy(), blocks)


@pytest.mark.parametrize("M,K,N", [(1, 256, 1), (13, 512, 2), (1000, 3584, 4), (37, 2048, 3),
                                   (3584, 18944, 1), (4096, 3584, 2), (33, 256, 1),
                                   (4739, 2304, 1), (70, 4864, 2), (5000, 1024, 2),
                                   # several tiles per CTA: the partial-sum buffers and
                                   # their barriers go round more than once
                                   (30000, 512, 1), (20000, 768, 2), (20000, 768, 3)])
def test_q6k_packed_gemv_matches_oracle(M, K, N):
    blocks = q8gen.kquant_matrix("q6_k", 5 * M + K + N, M, K)
    x = q8gen.activations(M + 2 * K + N, N, K)
    y = run_q6k_packed(pack_q6k(blocks, M, K), x, M, K)
    y_ref, y_abs = oracle.kquant_gemv("q6_k", blocks, x, M, K, threads=oracle.max_threads())
    assert_within(y, y_ref, TOL_REL * y_abs, f"q6_k packed M={M} K={K} N={N}")


@pytest.mark.parametrize("M,K,N", [(30000, 512, 1), (20000, 768, 2)])
def test_q4k_tile_many_tiles_per_cta(M, K, N):
    blocks = q8gen.kquant_matrix("q4_k", 7 * M + K, M, K)
    x = q8gen.activations(M + K + N, N, K)
    y = run("q4_k", blocks, x, M, K)
    y_ref, y_abs = oracle.kquant_gemv("q4_k", blocks, x, M, K, threads=oracle.max_threads())
    assert_within(y, y_ref, TOL_REL * y_abs, f"q4_k M={M} K={K} N={N}")


def test_q6k_packed_full_size_sampled_and_deterministic():
    """152064 x 3584 at N = 1 and 2 from the packed units, sampled rows; two
    runs bit-identical."""
    M, K = 152064, 3584
    blocks = q8gen.kquant_matrix("q6_k", 779, M, K)
    packed = pack_q6k(blocks, M, K)
    rows = np.unique(np.concatenate([np.arange(4), np.arange(M - 4, M),
                                     np.random.default_rng(1).integers(0, M, 200)]))
    sub = blocks.reshape(M, (K // 256) * 210)[rows].reshape(-1)
    for N in (1, 2):
        x = q8gen.activations(780 + N, N, K)
        y = run_q6k_packed(packed, x, M, K)
        assert np.array_equal(y, run_q6k_packed(packed, x, M, K))
        y_ref, y_abs = oracle.kquant_gemv("q6_k", sub, x, len(rows), K, threads=oracle.max_threads())
        assert_within(y[:, rows], y_ref, TOL_REL * y_abs, f"q6_k packed full size N={N}")


def test_q6k_packed_rejections():
    t = torch()
    M, K = 64, 512
    packed = t.zeros((q8().q8_q6k_packed_bytes(M, K),), dtype=t.uint8, device="cuda")
    y = t.empty((5, M), dtype=t.float32, device="cuda")
    assert q8().q8_q6k_packed_bytes(M, 300) == 0
    with pytest.raises(q8().Q8Error) as e:
        q8().q8_q6k_gemv_packed(packed, dev(np.zeros((5, K), np.float32)), y, M, K, 5)  # N > 4
    assert e.value.status == 5
    with pytest.raises(q8().Q8Error) as e:
        q8().q8_q6k_gemv_packed(packed[1:], dev(np.zeros((1, K), np.float32)), y, M, K, 1)  # unaligned
    assert e.value.status == 3
