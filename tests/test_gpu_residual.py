"""GPU parity of q8_gemv_residual (y = W x + residual, the residual-stream add
fused into the GEMV's store) against the fp64 oracle, through the C ABI, on
every kernel that serves q8_gemv: the resident kernel (small matrices, N = 1),
the column-owner kernel (N <= 4), and the tensor-core kernel (5 <= N <= 16).

Two checks per case: the output is one fp32 rounding of q8_gemv's own value
plus the residual (bit for bit), and it is within the GEMV bound of the exact
y + residual (plus that rounding)."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from q8_test_utils import TOL_REL, assert_within, dev, gemv, matrix, pack, torch

pytestmark = pytest.mark.gpu


def q8():
    import q8_block_quantized_02_b200 as m
    return m


@pytest.mark.parametrize("M,K,N", [(896, 896, 1), (896, 4864, 1), (4096, 896, 1), (151936, 896, 1), (1000, 2048, 2),
                                   (4096, 3584, 4), (1152, 896, 8), (3584, 18944, 16), (203, 1408, 5)])
@pytest.mark.parametrize("in_place", [False, True])
def test_gemv_residual_matches_oracle(M, K, N, in_place):
    t = torch()
    g, x = matrix(91 * M + K + N, M, K, N)
    res = np.random.default_rng(M + N).standard_normal((N, M)).astype(np.float32) * 4
    p = pack(g, M, K)
    r_dev = dev(res)
    y = r_dev if in_place else t.full((N, M), float("nan"), dtype=t.float32, device="cuda")
    q8().q8_gemv_residual(p, dev(x), r_dev, y, M, K, N)
    out = y.cpu().numpy()
    plain = gemv(p, x, M, K)
    assert np.array_equal(out, (plain + res).astype(np.float32))  # one fp32 rounding of the same value
    y_ref, y_abs = oracle.gemv_residual(g, x, res, M, K, threads=oracle.max_threads())
    assert_within(out, y_ref, TOL_REL * y_abs + 2.0 ** -23 * np.abs(y_ref), f"residual M={M} K={K} N={N}")
