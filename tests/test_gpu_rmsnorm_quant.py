"""GPU parity of q8_rmsnorm_quantize_act (RMSNorm fused in front of the Q8_0
activation quantiser, the prologue of the integer product) against the CPU
oracle, through the C ABI.

The per-row factor r is checked against the exact fp64 value within the
header's bound, (K/256 + 12) * 2^-24 relative; the quantised codes and scales -- integers decided by floating
point -- are checked bit for bit against the oracle fed the kernel's own r, so
both sides decide them in the same precision.  The chain RMSNorm -> quantise ->
Q8 x Q8 product is checked end to end against the oracle's integer product."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import q8gen
from q8_test_utils import TOL_REL, assert_within, dev, matrix, pack, torch

pytestmark = pytest.mark.gpu


def q8():
    import q8_block_quantized_02_b200 as m
    return m


def run(x, gamma, eps, with_r=True):
    t = torch()
    N, K = x.shape
    xq = t.empty((N, K), dtype=t.int8, device="cuda")
    xd = t.empty((N, K // 32), dtype=t.int16, device="cuda")
    r = t.full((N,), float("nan"), dtype=t.float32, device="cuda") if with_r else None
    q8().q8_rmsnorm_quantize_act(dev(x), dev(gamma), eps, xq, xd, r, N, K)
    return (xq.cpu().numpy(), xd.cpu().numpy().view(np.uint16),
            r.cpu().numpy() if with_r else None)


def r_bound(K):
    """Relative bound on the kernel's r stated in include/q8.h."""
    return (K / 256 + 12) * 2.0 ** -24


def gain(K, seed):
    rng = np.random.default_rng(seed)
    g = (1 + 0.2 * rng.standard_normal(K)).astype(np.float32)
    g[::97] = 0.0      # a few zero gains
    g[5::131] *= -1.0  # and some negative ones
    return g


@pytest.mark.parametrize("N,K", [(1, 896), (3, 3584), (16, 4864), (2, 32), (5, 18944), (7, 2048)])
def test_rmsnorm_quantize_matches_oracle(N, K):
    x = q8gen.activations(70 + N + K, N, K)
    x[0, :64] *= 50.0  # an outlier stretch in row 0
    g = gain(K, K)
    xq, xd, r = run(x, g, 1e-6)
    r_exact, _, q_ref, d_ref, _ = oracle.rmsnorm_quantize_act(x, g, 1e-6, r=r)
    assert np.all(np.abs(r - r_exact) <= r_bound(K) * r_exact)
    assert np.array_equal(xq, q_ref)
    assert np.array_equal(xd, d_ref)


def test_rmsnorm_quantize_without_r_and_zero_rows():
    N, K = 4, 1408
    x = q8gen.activations(71, N, K)
    x[2] = 0.0  # a zero row: r = 1/sqrt(eps), all codes and scales zero
    g = gain(K, 3)
    xq, xd, r = run(x, g, 1e-5)
    xq2, xd2, _ = run(x, g, 1e-5, with_r=False)
    assert np.array_equal(xq, xq2) and np.array_equal(xd, xd2)
    assert np.all(xq[2] == 0) and np.all(xd[2] == 0)
    assert abs(r[2] - 1e-5 ** -0.5) <= r_bound(K) * 1e-5 ** -0.5


def test_rmsnorm_quantize_feeds_the_integer_product():
    """RMSNorm -> quantise -> q8q8_gemv against the oracle's integer product on
    the same codes (its tolerance), for a 7B-class gate_up slice."""
    t = torch()
    M, K, N = 1024, 3584, 4
    g_w, _ = matrix(72, M, K)
    x = q8gen.activations(73, N, K)
    gam = gain(K, 4)
    xq, xd, r = run(x, gam, 1e-6)
    y = t.empty((N, M), dtype=t.float32, device="cuda")
    q8().q8q8_gemv(pack(g_w, M, K), dev(xq), dev(xd.view(np.int16)), y, M, K, N)
    _, y_ref, y_abs = oracle.q8q8(g_w, xq, xd, M, K, want_dots=False, threads=oracle.max_threads())
    assert_within(y.cpu().numpy(), y_ref, TOL_REL * y_abs, "rmsnorm -> q8q8")


def test_rmsnorm_quantize_rejects_bad_eps():
    t = torch()
    x = np.ones((1, 32), np.float32)
    xq = t.empty((1, 32), dtype=t.int8, device="cuda")
    xd = t.empty((1, 1), dtype=t.int16, device="cuda")
    for eps in (-1e-6, float("nan"), float("inf")):
        with pytest.raises(q8().Q8Error) as e:
            q8().q8_rmsnorm_quantize_act(dev(x), dev(np.ones(32, np.float32)), eps, xq, xd, None, 1, 32)
        assert e.value.status == 1


def _boundary_margin(x, gamma, eps, r_exact):
    """For every element, the distance of the exact x_hat / d (fp64: x * r_exact
    * gamma over amax / 127 of its block) from the nearest half-integer, the
    points where round-half-away changes the code, and the exact value itself."""
    N, K = x.shape
    xh = x.astype(np.float64) * r_exact[:, None] * gamma.astype(np.float64)[None, :]
    blocks = xh.reshape(N, K // 32, 32)
    amax = np.abs(blocks).max(axis=2, keepdims=True)
    with np.errstate(invalid="ignore", divide="ignore"):
        v = np.where(amax > 0, blocks / (amax / 127.0), 0.0).reshape(N, K)
    dist = np.abs(np.abs(v) - (np.floor(np.abs(v)) + 0.5))
    return v, dist


@pytest.mark.parametrize("N,K", [(1, 896), (4, 3584), (16, 4864), (2, 18944)])
def test_rmsnorm_codes_against_exact_r(N, K):
    """The codes checked against an oracle that does not see the kernel's r:
    codes taken from r_exact rounded to fp32.  Both sides round x_hat = (x r) g
    and x_hat / d in fp32, so a code may differ only where the exact x_hat / d
    sits within the propagated error of a rounding boundary: the kernel's r
    within (K/256 + 12) 2^-24 of the exact value, plus the fp32 roundings of
    x r, of the gain product, of amax / 127 and of the division (a few
    2^-24 each).  Every differing code must be such an element, and they must
    be rare; the scales may differ only where d = amax / 127 lies that close to
    a binary16 rounding midpoint."""
    x = q8gen.activations(170 + N + K, N, K)
    x[0, :64] *= 50.0
    g = gain(K, K + 1)
    eps = 1e-6
    xq, xd, r = run(x, g, eps)
    r_exact, _, q_ref, d_ref, d32_ref = oracle.rmsnorm_quantize_act(x, g, eps)  # r = fp32(r_exact)
    assert np.all(np.abs(r - r_exact) <= r_bound(K) * r_exact)
    v, dist = _boundary_margin(x, g, eps, r_exact)
    rel = 2 * r_bound(K) + 8 * 2.0 ** -24
    near = dist <= rel * np.abs(v) + 2.0 ** -20
    diff = xq != q_ref
    assert not np.any(diff & ~near), (
        f"{int((diff & ~near).sum())} codes differ away from any rounding boundary")
    assert np.all(np.abs(xq.astype(np.int32) - q_ref.astype(np.int32)) <= 1)
    assert diff.sum() <= max(2, diff.size // 1000)
    # binary16 scales: equal unless d sits next to a rounding midpoint
    dd = xd != d_ref
    if dd.any():
        d16 = d_ref.view(np.float16).astype(np.float64)
        ulp = np.spacing(np.abs(d_ref.view(np.float16))).astype(np.float64)
        mid_dist = np.abs(np.abs(d32_ref.astype(np.float64) - d16) - ulp / 2)
        assert np.all(mid_dist[dd] <= (rel + 2.0 ** -23) * np.abs(d32_ref[dd]))
