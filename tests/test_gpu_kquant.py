"""GPU parity of the K-quant GEMV (q8_q4k_gemv, q8_q6k_gemv: GGUF Q4_K / Q6_K
super-blocks read in their raw layout) against the fp64 CPU oracle, through
the C ABI.  Every packed field is random bytes, so all scale/min bit patterns
and all nibble values occur.

Tolerance: |y - y_ref| <= 1e-5 * sum_k |w_k x_k| per element, the GEMV bar."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import q8gen
from q8_test_utils import TOL_REL, assert_within, dev, torch

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
                                   (3584, 18944, 1), (4096, 3584, 2)])
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
