"""GPU parity of the resident GEMV kernel (small matrices at N = 1) against
the fp64 oracle, across its planning regimes: one row group per CTA, several
row groups per CTA (CTAs holding TGM or TGM - 1 of them), one or two column
chunks, the SwiGLU pair, ragged last groups, and shapes too large for it (the
column kernel takes them).  Also a
chain of dependent launches on one stream, as a decode step issues them."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from q8_test_utils import TOL_REL, assert_within, dev, gate_up, gemv, matrix, pack, swiglu_bound, torch

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K", [
    (1152, 896),    # 144 groups on 144 CTAs, 56 columns
    (896, 4864),    # 304 columns in two chunks of 160 (the second one zero-filled past K)
    (100, 8192),    # 512 columns (too large: column kernel)
    (100, 6144),    # 13 groups, 384 columns
    (1157, 896),    # ragged last group (5 rows)
    (2000, 896),    # 250 groups: two per CTA on most CTAs
    (6000, 1408),   # six groups per CTA
    (9000, 896),    # eight groups per CTA
    (1200, 4608),   # two chunks of 144 columns, one or two groups per CTA
    (9000, 4864),   # too large for shared memory: column kernel
])
def test_resident_gemv_matches_oracle(M, K):
    g, x = matrix(M + 3 * K, M, K, 1)
    y = gemv(pack(g, M, K), x, M, K)
    y_ref, y_abs = oracle.gemv(g, x, M, K, threads=oracle.max_threads())
    assert_within(y, y_ref, TOL_REL * y_abs, f"resident gemv {M}x{K}")


@pytest.mark.parametrize("I,K", [
    (4864, 896),    # 608 gate groups: four or five per CTA
    (1408, 2048),   # two groups per CTA, 128 columns
    (104, 4864),    # one gate group per CTA, 304 columns (column kernel: over the shared-memory budget)
    (2400, 1024),   # three groups per CTA
    (160, 4608),    # two chunks of 144 columns, gate and up
    (9000, 896),    # too large for shared memory: column kernel
])
def test_resident_swiglu_matches_oracle(I, K):
    g, x = matrix(I + 5 * K, 2 * I, K, 1)
    h = gate_up(pack(g, 2 * I, K), x, I, K)
    ref = oracle.gate_up_swiglu(g, x, I, K, threads=oracle.max_threads())
    assert_within(h, ref["h"], swiglu_bound(ref), f"resident swiglu I={I} K={K}")


def test_resident_dependent_chain():
    """y of one launch is x of the next, on one stream with no host sync in
    between: each launch must read its input only after the previous grid
    is done (programmatic dependent launch), and the chain must equal the
    oracle applied step by step to the GPU's own intermediate values."""
    import q8_block_quantized_02_b200 as q8
    t = torch()
    K = 896
    mats = [matrix(40 + i, K, K, 1)[0] for i in range(6)]
    packed = [pack(g, K, K) for g in mats]
    x0 = matrix(99, 8, K, 1)[1]
    bufs = [dev(x0)] + [t.full((1, K), float("nan"), dtype=t.float32, device="cuda") for _ in mats]
    for i in range(len(mats)):
        q8.q8_gemv(packed[i], bufs[i], bufs[i + 1], K, K, 1)
    outs = [b.cpu().numpy() for b in bufs]
    for i, g in enumerate(mats):
        y_ref, y_abs = oracle.gemv(g, outs[i].astype(np.float32), K, K)
        assert_within(outs[i + 1], y_ref, TOL_REL * y_abs, f"chain step {i}")
