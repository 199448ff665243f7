"""GPU parity of q8_gemv_argmax, the Q8_0 GEMV with the arg-max over its
outputs fused in (greedy decoding's last step), through the C ABI.

The pick is an integer decided by floating point, so it is compared in the
kernel's own precision: it must equal the first maximum of the fp32 logits the
same call writes, those logits must meet the GEMV tolerance against the fp64
oracle (and equal q8_gemv's bits where q8_gemv takes the same kernel), and the
pick must be valid against the oracle -- its exact logit within the GEMV
tolerance of the exact maximum.  Ties (duplicated rows) must go to the lowest
index."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from q8_test_utils import TOL_REL, assert_within, dev, gemv, matrix, pack, torch

pytestmark = pytest.mark.gpu


def q8():
    import q8_block_quantized_02_b200 as m
    return m


def argmax_gpu(packed, x, M, K, with_y=True):
    t = torch()
    N = x.shape[0]
    xd = dev(x.astype(np.float32))
    y = t.full((N, M), float("nan"), dtype=t.float32, device="cuda") if with_y else None
    best = t.full((N,), -1, dtype=t.int64, device="cuda")  # the call zeroes it first
    q8().q8_gemv_argmax(packed, xd, y, M, K, N, best)
    keys = best.cpu().numpy().view(np.uint64)
    return q8().q8_argmax_index(keys), q8().q8_argmax_value(keys), (y.cpu().numpy() if with_y else None)


def check_against_oracle(g, x, M, K, idx):
    _, y_ref, y_abs = oracle.gemv_argmax(g, x, M, K, threads=oracle.max_threads())
    tol = TOL_REL * y_abs
    for n in range(x.shape[0]):
        m_ref = int(np.argmax(y_ref[n]))
        # the pick's exact logit is within the two outputs' tolerances of the exact maximum
        assert y_ref[n, idx[n]] >= y_ref[n, m_ref] - tol[n, idx[n]] - tol[n, m_ref], (n, idx[n], m_ref)


@pytest.mark.parametrize("M,K,N", [(151936, 896, 1), (1000, 2048, 2), (13, 32, 3), (4096, 3584, 4),
                                   (1153, 896, 1), (203, 1408, 4)])
def test_argmax_matches_own_logits_and_oracle(M, K, N):
    g, x = matrix(61 * M + K + N, M, K, N)
    p = pack(g, M, K)
    idx, val, y = argmax_gpu(p, x, M, K)
    assert np.array_equal(idx, np.argmax(y, axis=1))  # first maximum of its own fp32 logits
    assert np.array_equal(val, y[np.arange(N), idx])
    y_ref, y_abs = oracle.gemv(g, x, M, K, threads=oracle.max_threads())
    assert_within(y, y_ref, TOL_REL * y_abs, f"argmax logits M={M} K={K} N={N}")
    if M > 148 * 64:  # beyond the resident kernel's reach q8_gemv takes the same column-owner kernel
        assert np.array_equal(y, gemv(p, x, M, K))
    check_against_oracle(g, x, M, K, idx)


def test_argmax_without_logits():
    M, K, N = 5000, 896, 2
    g, x = matrix(404, M, K, N)
    p = pack(g, M, K)
    idx0, val0, _ = argmax_gpu(p, x, M, K, with_y=True)
    idx1, val1, _ = argmax_gpu(p, x, M, K, with_y=False)
    assert np.array_equal(idx0, idx1) and np.array_equal(val0, val1)


def test_argmax_ties_go_to_the_lowest_index():
    """Copies of the winning row placed before and after it (other CTAs' ranges
    too): the earliest copy wins."""
    M, K, N = 6000, 896, 1
    g, x = matrix(505, M, K, N)
    B = K // 32
    rows = g.reshape(M, B * 34).copy()
    top = int(np.argmax(gemv(pack(g, M, K), x, M, K)[0]))
    for r in (17, 2999, 5998):
        rows[r] = rows[top]
    g2 = rows.reshape(-1)
    idx, _, y = argmax_gpu(pack(g2, M, K), x, M, K)
    want = min(17, top)
    assert y[0, want] == y[0].max()
    assert idx[0] == want


def test_argmax_all_negative_logits():
    """Non-negative q against non-positive x: every logit is <= 0, so the pick
    is the logit nearest zero (the sign-flipped half of the key order)."""
    import q8gen
    M, K, N = 3000, 896, 3
    g, x = matrix(606, M, K, N)
    q, dbits = q8gen.split_gguf(g, M, K)
    g_pos = q8gen.assemble_gguf(np.abs(q.astype(np.int16)).astype(np.int8), dbits)
    x_neg = -np.abs(x)
    p = pack(g_pos, M, K)
    idx, val, y = argmax_gpu(p, x_neg, M, K)
    assert np.all(y <= 0)
    assert np.array_equal(idx, np.argmax(y, axis=1))
    assert np.array_equal(val, y[np.arange(N), idx])
    check_against_oracle(g_pos, x_neg, M, K, idx)


def test_argmax_rejects_wide_batches():
    m = q8()
    t = torch()
    M, K = 16, 64
    g, x = matrix(1, M, K, 5)
    p = pack(g, M, K)
    best = t.zeros(5, dtype=t.int64, device="cuda")
    with pytest.raises(m.Q8Error) as e:
        m.q8_gemv_argmax(p, dev(x), None, M, K, 5, best)
    assert e.value.status == 5
