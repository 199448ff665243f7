"""CPU pins of the three-term int8 split of fp32 activations that the
tensor-core path for 5 <= N <= 16 uses (q8_gemv / q8_gate_up_swiglu).

Per 32-block with amax = max|x|, s is the power of two with amax/s in
[32, 64), v0 = x/s, q0 = rint(v0), v1 = (v0 - q0)*254, q1 = rint(v1),
v2 = (v1 - q1)*254, q2 = rint(v2), every step an IEEE fp32 operation (the
kernel uses unfused adds and multiplies, rint by adding and subtracting
1.5*2^23).  Claimed, and checked here in numpy float32 on blocks of many kinds:
the pieces fit int8 (|q0| <= 64, |q1|, |q2| <= 127); x = s*(q0 + q1/254 +
q2/254^2) to within 2.5e-7 of amax; x -> 2x gives the same pieces and twice s;
a unit block (one 1, the rest 0) splits exactly.  These are the properties the
GPU tolerance and its exact-scaling and one-hot tests rely on."""
from __future__ import annotations

import numpy as np

F = np.float32
MAGIC = F(12582912.0)  # 1.5 * 2^23


def split(xb: np.ndarray):
    xb = xb.astype(F)
    amax = F(np.max(np.abs(xb)))
    e = max((int(amax.view(np.uint32)) >> 23) & 0xFF, 6)
    s = np.uint32((e - 5) << 23).view(F)
    inv = np.uint32((259 - e) << 23).view(F)
    v = (xb * inv).astype(F)
    pieces = []
    for k in range(3):
        t = (v + MAGIC).astype(F)
        q = (t - MAGIC).astype(F)
        low = (t.view(np.uint32) & 0xFF).astype(np.int32)
        low = np.where(low > 127, low - 256, low)
        assert np.array_equal(low, q.astype(np.int32))  # the stored byte is rint(v) as int8
        pieces.append(q.astype(np.int64))
        if k < 2:
            v = ((v - q).astype(F) * F(254)).astype(F)
    return s, pieces, amax


def blocks(rng, count):
    for i in range(count):
        kind = i % 5
        x = rng.standard_normal(32).astype(F)
        if kind == 1:                     # tiny values with one large one
            x = (x * F(1e-7)).astype(F)
            x[rng.integers(32)] = F(3e4)
        elif kind == 2:                   # a wide range of block magnitudes
            x = (x * F(10.0) ** rng.integers(-30, 31)).astype(F)
        elif kind == 3:                   # exact ties for rint
            x[:] = F(rng.choice([127.0, 1.0, 0.5, 63.99]))
            x[1::2] *= F(-0.5)
        elif kind == 4:                   # heavy tails
            x = (rng.standard_cauchy(32)).astype(F)
        yield x


def test_split_ranges_and_residual_bound():
    rng = np.random.default_rng(2024)
    worst = 0.0
    for xb in blocks(rng, 5000):
        s, (q0, q1, q2), amax = split(xb)
        assert np.abs(q0).max() <= 64 and np.abs(q1).max() <= 127 and np.abs(q2).max() <= 127
        rep = np.float64(s) * (q0 + q1 / 254.0 + q2 / 254.0 ** 2)
        if amax > 0:
            worst = max(worst, float(np.max(np.abs(rep - xb.astype(np.float64))) / amax))
    assert worst < 2.5e-7


def test_split_is_exact_under_powers_of_two():
    rng = np.random.default_rng(7)
    for xb in blocks(rng, 500):
        if np.max(np.abs(xb)) > 1e30 or np.max(np.abs(xb)) < 1e-30:
            continue  # keep 2x and x/2 inside the normal fp32 range
        s1, p1, _ = split(xb)
        s2, p2, _ = split((xb * F(2)).astype(F))
        assert s2 == 2 * s1 and all(np.array_equal(a, b) for a, b in zip(p1, p2))


def test_unit_block_splits_exactly():
    x = np.zeros(32, F)
    x[5] = 1.0
    s, (q0, q1, q2), _ = split(x)
    assert s * q0[5] == 1.0 and not q1.any() and not q2.any()
