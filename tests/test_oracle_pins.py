"""Pins for the CPU oracle: each check fixes the oracle to something other than
itself -- hand-computed fixtures, closed forms, invariants, exact rational brute
force, and library conversions -- so that a dropped term, a wrong sign or
index, or a transposed operand anywhere in the oracle fails one of them.
CPU only."""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import q8gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# binary16 conversions, pinned to numpy's float16 (a library routine)
# --------------------------------------------------------------------------

def test_half_decode_matches_numpy_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # signed zero survives
    assert math.copysign(1.0, oracle.half_to_double(0x8000)) == -1.0


def _encode_cases():
    rng = np.random.default_rng(7)
    halves = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    mids = (halves[:-1] + halves[1:]) / 2  # exact ties between neighbours
    vals = np.concatenate([
        halves, mids, np.nextafter(mids, 0), np.nextafter(mids, 1),
        rng.standard_normal(20000) * 0.02,
        np.exp(rng.uniform(-20, 11.2, 20000)),
        [65504, 65519.99, 65520, 65536, 1e9, 2.0 ** -24, 2.0 ** -25, 2.0 ** -26, 3 * 2.0 ** -26],
    ])
    vals = vals.astype(np.float32)
    return np.concatenate([vals, -vals])


def test_half_encode_matches_numpy():
    vals = _encode_cases()
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float16).view(np.uint16)
    got = np.array([oracle.float_to_half_rn(float(v)) for v in vals], np.uint16)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, f"{bad.size} mismatches, e.g. {vals[bad[:5]]}"


# --------------------------------------------------------------------------
# GGUF block layout (hand-written bytes)
# --------------------------------------------------------------------------

def _read_layout():
    entries, cur = [], {}
    for line in open(os.path.join(GOLDEN, "q8_0_block_layout.txt")):
        if line.startswith("#") or not line.strip():
            continue
        key, val = line.split(":", 1)
        cur[key.strip()] = val.split()
        if key.strip() == "q":
            entries.append(cur)
            cur = {}
    return entries


def test_block_layout_decodes_as_written():
    for e in _read_layout():
        raw = np.array([int(b, 16) for b in e["bytes"]], np.uint8)
        assert raw.size == 34
        d = float(e["d"][0])
        q = np.array([int(v) for v in e["q"]], np.int64)
        # Decode through the oracle's GEMV with one-hot activations: y_k = d * q_k.
        for k in range(32):
            x = np.zeros((1, 32), np.float32)
            x[0, k] = 1.0
            y, _ = oracle.gemv(raw, x, 1, 32)
            assert y[0, 0] == d * q[k]
        # ...and the generator's assembler writes the same bytes back.
        dbits = np.array([[int(raw[0]) | (int(raw[1]) << 8)]], np.uint16)
        again = q8gen.assemble_gguf(q.astype(np.int8).reshape(1, 32), dbits)
        assert np.array_equal(again, raw)


# --------------------------------------------------------------------------
# P5: hand-computed blocks
# --------------------------------------------------------------------------

def _hand_blocks():
    out = []
    for line in open(os.path.join(GOLDEN, "hand_blocks.txt")):
        if line.startswith("#") or not line.strip():
            continue
        d, q, x, y = [p.split() for p in line.split("|")]
        out.append((float(d[0]), [int(v) for v in q], [float(v) for v in x], float(y[0])))
    return out


@pytest.mark.parametrize("case", range(4))
def test_hand_blocks(case):
    d, q, x, y = _hand_blocks()[case]
    dbits = np.array([[np.float16(d).view(np.uint16)]], np.uint16)
    g = q8gen.assemble_gguf(np.array([q], np.int8), dbits)
    got, gabs = oracle.gemv(g, np.array([x], np.float32), 1, 32)
    assert got[0, 0] == y
    assert gabs[0, 0] == sum(abs(d * qi * xi) for qi, xi in zip(q, x))


# --------------------------------------------------------------------------
# P1: brute force with exact rationals on tiny shapes
# --------------------------------------------------------------------------

def _exact_gemv(gguf, x, M, K):
    q, dbits = q8gen.split_gguf(gguf, M, K)
    d = dbits.view(np.float16).astype(np.float64)
    N = x.shape[0]
    y = [[Fraction(0)] * M for _ in range(N)]
    for n in range(N):
        for m in range(M):
            s = Fraction(0)
            for k in range(K):
                s += Fraction(float(d[m, k // 32])) * int(q[m, k]) * Fraction(float(x[n, k]))
            y[n][m] = s
    return y


@pytest.mark.parametrize("M,K,N,seed", [(1, 32, 1, 1), (3, 64, 2, 2), (4, 32, 3, 3), (2, 96, 1, 4)])
def test_brute_force_gemv(M, K, N, seed):
    g, x = q8gen.q8_matrix(seed, M, K, N)
    y, ya = oracle.gemv(g, x, M, K)
    exact = _exact_gemv(g, x, M, K)
    for n in range(N):
        for m in range(M):
            e = exact[n][m]
            assert abs(Fraction(y[n, m]) - e) <= Fraction(ya[n, m]) * Fraction(2, 2 ** 52)


def test_brute_force_gate_up_g_u():
    I, K = 3, 64
    g8, x = q8gen.q8_matrix(11, 2 * I, K, 2)
    out = oracle.gate_up_swiglu(g8, x, I, K)
    exact = _exact_gemv(g8, x, 2 * I, K)
    for n in range(2):
        for i in range(I):
            assert abs(Fraction(out["g"][n, i]) - exact[n][i]) <= Fraction(out["g_abs"][n, i]) / 2 ** 51
            assert abs(Fraction(out["u"][n, i]) - exact[n][I + i]) <= Fraction(out["u_abs"][n, i]) / 2 ** 51


def test_brute_force_q8q8():
    M, K, N = 3, 64, 2
    g, x = q8gen.q8_matrix(21, M, K, N)
    xq, xd, _ = oracle.quantize_act(x)
    dots, y, ya = oracle.q8q8(g, xq, xd, M, K)
    q, dbits = q8gen.split_gguf(g, M, K)
    dw = dbits.view(np.float16).astype(np.float64)
    dx = xd.view(np.float16).astype(np.float64)
    for n in range(N):
        for m in range(M):
            tot = Fraction(0)
            for b in range(K // 32):
                dot = sum(int(q[m, b * 32 + i]) * int(xq[n, b * 32 + i]) for i in range(32))
                assert dots[n, m, b] == dot
                tot += Fraction(float(dw[m, b])) * Fraction(float(dx[n, b])) * dot
            assert abs(Fraction(y[n, m]) - tot) <= Fraction(ya[n, m]) / 2 ** 51


# --------------------------------------------------------------------------
# P2: closed form -- unit scales and one-hot x return a column of q exactly
# --------------------------------------------------------------------------

def test_one_hot_returns_column():
    M, K = 5, 96
    rng = np.random.default_rng(5)
    q = rng.integers(-127, 128, (M, K), dtype=np.int8)
    dbits = np.full((M, K // 32), 0x3C00, np.uint16)  # d = 1.0
    g = q8gen.assemble_gguf(q, dbits)
    for k in (0, 31, 32, 95):
        x = np.zeros((1, K), np.float32)
        x[0, k] = 1.0
        y, _ = oracle.gemv(g, x, M, K)
        assert np.array_equal(y[0], q[:, k].astype(np.float64))


def test_row_and_column_orientation():
    """x column n and output row m are not transposed: distinct rows and
    distinct activation vectors give distinct, correctly placed results."""
    M, K = 2, 32
    q = np.zeros((M, K), np.int8)
    q[0, 0] = 1      # row 0 picks x[:, 0]
    q[1, 1] = 1      # row 1 picks x[:, 1]
    g = q8gen.assemble_gguf(q, np.full((M, 1), 0x3C00, np.uint16))
    x = np.zeros((3, K), np.float32)
    x[:, 0] = [1, 2, 3]
    x[:, 1] = [10, 20, 30]
    y, _ = oracle.gemv(g, x, M, K)
    assert np.array_equal(y, [[1, 10], [2, 20], [3, 30]])


def test_argmax_closed_forms():
    """O8 against brute force: with unit scales and one-hot x the outputs are a
    column of q, so the pick is found by scanning that column for its first
    maximum by hand; equal rows give the earliest; all-negative columns pick
    the value nearest zero; several activation rows pick independently."""
    M, K = 40, 64
    rng = np.random.default_rng(17)
    q = rng.integers(-127, 128, (M, K), dtype=np.int8)
    q[3, 5] = q[21, 5] = q[33, 5] = 127          # three-way tie at the maximum of column 5
    q[:, 9] = -rng.integers(1, 128, M)           # column 9 all negative
    q[:, 9][[11, 30]] = -1                       # ... its maximum (-1) twice
    g = q8gen.assemble_gguf(q, np.full((M, K // 32), 0x3C00, np.uint16))
    cols = [5, 9, 0, 63]
    x = np.zeros((len(cols), K), np.float32)
    for n, k in enumerate(cols):
        x[n, k] = 1.0
    idx, y, _ = oracle.gemv_argmax(g, x, M, K)
    for n, k in enumerate(cols):
        best = 0
        for m in range(1, M):
            if int(q[m, k]) > int(q[best, k]):
                best = m
        assert idx[n] == best
    assert idx[0] == 3 and idx[1] == 11


# --------------------------------------------------------------------------
# P3: linearity in d and x
# --------------------------------------------------------------------------

def test_linearity():
    M, K = 7, 128
    g, x = q8gen.q8_matrix(31, M, K, 2)
    y, ya = oracle.gemv(g, x, M, K)
    # doubling every d (exact in binary16 away from the top of the range)
    q, dbits = q8gen.split_gguf(g, M, K)
    d2 = (dbits.view(np.float16).astype(np.float32) * 2).astype(np.float16).view(np.uint16)
    y2, _ = oracle.gemv(q8gen.assemble_gguf(q, d2), x, M, K)
    assert np.array_equal(y2, 2 * y)
    # doubling x
    y3, _ = oracle.gemv(g, 2 * x, M, K)
    assert np.array_equal(y3, 2 * y)
    # additivity
    xa = q8gen.activations(1, 2, K)
    xb = q8gen.activations(2, 2, K)
    ya_, aa = oracle.gemv(g, xa, M, K)
    yb_, ab = oracle.gemv(g, xb, M, K)
    xs = (xa.astype(np.float64) + xb).astype(np.float32)
    ys, _ = oracle.gemv(g, xs, M, K)
    # x_a + x_b is rounded to fp32 once per element: bound that, plus fp64 sums
    rounding = oracle.gemv(q8gen.assemble_gguf(np.abs(q.astype(np.int16)).astype(np.int8), dbits),
                           np.abs(xs), M, K)[0] * 2.0 ** -24
    assert np.all(np.abs(ys - (ya_ + yb_)) <= rounding + 1e-12 * (aa + ab))
    # negating q flips the sign exactly
    yn, _ = oracle.gemv(q8gen.assemble_gguf(-q, dbits), x, M, K)
    assert np.array_equal(yn, -y)


# --------------------------------------------------------------------------
# P4: Q8_0 round trip |w - d*q| <= d/2
# --------------------------------------------------------------------------

def test_round_trip_bound():
    rng = np.random.default_rng(9)
    M, K = 16, 256
    w = (rng.standard_normal((M, K)) * np.exp(rng.uniform(-8, 4, (M, 1)))).astype(np.float32)
    w[3, 32:64] = 0.0  # an all-zero block
    gguf, d32 = oracle.quantize_weights(w)
    q, dbits = q8gen.split_gguf(gguf, M, K)
    d = np.repeat(d32.astype(np.float64), 32, axis=1)
    err = np.abs(w.astype(np.float64) - d * q)
    # d32 and w/d32 are fp32-rounded: allow their rounding on top of d/2
    assert np.all(err <= d / 2 * (1 + 2.0 ** -20))
    assert np.all(q[3, 32:64] == 0) and dbits[3, 1] == 0
    # the largest |w| of a block maps to +-127
    blk = np.abs(w.reshape(M, K // 32, 32)).argmax(axis=2)
    qb = np.abs(q.reshape(M, K // 32, 32))
    pick = np.take_along_axis(qb, blk[..., None], 2)[..., 0]
    nz = d32 > 0
    assert np.all(pick[nz] == 127)
    # stored scale is binary16(d32)
    assert np.array_equal(dbits, d32.astype(np.float16).view(np.uint16))


# --------------------------------------------------------------------------
# P6: activation quantisation -- hand blocks and invariants
# --------------------------------------------------------------------------

def _act_blocks():
    out = []
    for line in open(os.path.join(GOLDEN, "act_quant_blocks.txt")):
        if line.startswith("#") or not line.strip():
            continue
        x, q, d = [p.split() for p in line.split("|")]
        out.append((np.array([float(v) for v in x], np.float32), [int(v) for v in q], int(d[0], 16)))
    return out


def test_act_quant_hand_blocks():
    blocks = _act_blocks()
    x = np.stack([b[0] for b in blocks]).reshape(1, -1)
    q, d, _ = oracle.quantize_act(x)
    for i, (_, qq, dd) in enumerate(blocks):
        assert q[0, 32 * i:32 * (i + 1)].tolist() == qq
        assert int(d[0, i]) == dd


def test_act_quant_invariants():
    rng = np.random.default_rng(12)
    x = (rng.standard_normal((4, 4864)) * np.exp(rng.uniform(-30, 30, (4, 1)))).astype(np.float32)
    x[1, :64] = 0
    x[2, 100] = -np.float32(3.0e38)
    q, d, d32 = oracle.quantize_act(x)
    xb = x.reshape(4, -1, 32).astype(np.float64)
    qb = q.reshape(4, -1, 32).astype(np.float64)
    amax = np.abs(xb).max(axis=2)
    assert np.array_equal(d32, (amax.astype(np.float32) / np.float32(127)))
    dd = d32.astype(np.float64)[..., None]
    assert np.all(np.abs(xb - dd * qb) <= dd / 2 * (1 + 2.0 ** -20) + (dd == 0))
    assert np.all((np.sign(qb) == np.sign(xb)) | (qb == 0))
    assert np.all(np.abs(qb) <= 127)
    assert np.all(np.abs(qb).max(axis=2)[amax > 0] == 127)
    assert np.all(qb[1, :2] == 0) and np.all(d[1, :2] == 0)
    with np.errstate(over="ignore"):
        assert np.array_equal(d, d32.astype(np.float16).view(np.uint16))


# --------------------------------------------------------------------------
# P7: integer block dots
# --------------------------------------------------------------------------

# --------------------------------------------------------------------------
# O11: K-quant formats (Q4_K, Q6_K), against a packer written here from the
# stated layout (the inverse of the oracle's unpacking) and hand-computed blocks
# --------------------------------------------------------------------------

def _pack_q4k(d_bits, dmin_bits, sc, m, q):
    """One Q4_K block from 6-bit scales/mins sc[8], m[8] and nibbles q[256]."""
    b = np.zeros(144, np.uint8)
    b[0], b[1] = d_bits & 0xFF, d_bits >> 8
    b[2], b[3] = dmin_bits & 0xFF, dmin_bits >> 8
    for j in range(4):
        b[4 + j] = (sc[j] & 63) | ((sc[j + 4] >> 4) << 6)
        b[8 + j] = (m[j] & 63) | ((m[j + 4] >> 4) << 6)
        b[12 + j] = (sc[j + 4] & 15) | ((m[j + 4] & 15) << 4)
    for e in range(256):
        i = 16 + 32 * (e // 64) + e % 32
        b[i] |= (q[e] & 15) << (0 if e % 64 < 32 else 4)
    return b


def _pack_q6k(d_bits, scales, q):
    """One Q6_K block from int8 scales[16] and q[256] in [-32, 31]."""
    b = np.zeros(210, np.uint8)
    for e in range(256):
        u = int(q[e]) + 32
        h, c, l = e // 128, (e % 128) // 32, e % 32
        b[64 * h + 32 * (c & 1) + l] |= (u & 15) << (4 * (c >> 1))
        b[128 + 32 * h + l] |= (u >> 4) << (2 * c)
    b[192:208] = np.asarray(scales, np.int8).view(np.uint8)
    b[208], b[209] = d_bits & 0xFF, d_bits >> 8
    return b


def test_kquant_round_trip():
    """Random fields packed here decode, in the oracle, to exactly d*sc*q - dmin*m
    (Q4_K) and d*scale*q (Q6_K) at every position; the GEMV equals the fp64
    product of those weights."""
    rng = np.random.default_rng(31)
    for trial in range(6):
        dbits, mbits = [int(v) for v in (np.abs(rng.standard_normal(2)) * 0.01).astype(np.float16).view(np.uint16)]
        sc, m = rng.integers(0, 64, 8), rng.integers(0, 64, 8)
        q = rng.integers(0, 16, 256)
        blk4 = _pack_q4k(dbits, mbits, sc, m, q)
        d, dmin = oracle.half_to_double(dbits), oracle.half_to_double(mbits)
        want4 = np.array([d * sc[e // 32] * q[e] - dmin * m[e // 32] for e in range(256)])
        x = rng.standard_normal((2, 256)).astype(np.float32)
        y, _, w = oracle.kquant_gemv("q4_k", blk4, x, 1, 256, want_w=True)
        assert np.array_equal(w[0], want4)
        assert np.allclose(y[:, 0], x.astype(np.float64) @ want4, rtol=1e-12, atol=0)
        scales6 = rng.integers(-128, 128, 16)
        q6 = rng.integers(-32, 32, 256)
        blk6 = _pack_q6k(dbits, scales6, q6)
        want6 = np.array([d * scales6[e // 16] * q6[e] for e in range(256)])
        y6, _, w6 = oracle.kquant_gemv("q6_k", blk6, x, 1, 256, want_w=True)
        assert np.array_equal(w6[0], want6)
        assert np.allclose(y6[:, 0], x.astype(np.float64) @ want6, rtol=1e-12, atol=0)


def test_kquant_hand_blocks():
    """Q4_K: d = 1, dmin = 0.5; scales bytes give sc0 = 3, m0 = 1, sc4 = 53,
    m4 = 34 (high bits from bytes 0 and 4), all other scales and mins 0; every
    qs byte 0x21.  Sub-block 0 weights 1*3*1 - 0.5*1 = 2.5, sub-block 4 weights
    53*1 - 0.5*34 = 36, the rest 0: with x = 1, y = 32*2.5 + 32*36 = 1232.
    Q6_K: d = 0.25, scales[0] = -3, the others 2; ql bytes 0xFF, qh 0 (q = 15 -
    32 = -17): weights 12.75 (first 16) and -8.5: y = 204 - 2040 = -1836."""
    b = np.zeros(144, np.uint8)
    b[0:4] = [0x00, 0x3C, 0x00, 0x38]
    b[4] = 0b11000011   # sc0 = 3, top bits of sc4 = 3
    b[8] = 0b10000001   # m0 = 1, top bits of m4 = 2
    b[12] = 0x25        # sc4 low = 5, m4 low = 2
    b[16:] = 0x21
    y, _, w = oracle.kquant_gemv("q4_k", b, np.ones((1, 256), np.float32), 1, 256, want_w=True)
    assert y[0, 0] == 1232.0
    assert np.all(w[0, :32] == 2.5) and np.all(w[0, 128:160] == 36.0)
    assert np.all(w[0, 32:128] == 0) and np.all(w[0, 160:] == 0)
    b6 = np.zeros(210, np.uint8)
    b6[:128] = 0xFF
    b6[192:208] = np.array([-3] + [2] * 15, np.int8).view(np.uint8)
    b6[208:210] = [0x00, 0x34]
    y6, _ = oracle.kquant_gemv("q6_k", b6, np.ones((1, 256), np.float32), 1, 256)
    assert y6[0, 0] == -1836.0


def test_gemv_residual_closed_form():
    """O10: unit scales and one-hot x give a column of q, so y + residual is
    that column plus the residual, exactly."""
    M, K = 24, 64
    rng = np.random.default_rng(9)
    q = rng.integers(-127, 128, (M, K), dtype=np.int8)
    g = q8gen.assemble_gguf(q, np.full((M, K // 32), 0x3C00, np.uint16))
    x = np.zeros((2, K), np.float32)
    x[0, 7], x[1, 40] = 1.0, 1.0
    res = rng.standard_normal((2, M)).astype(np.float32)
    y, _ = oracle.gemv_residual(g, x, res, M, K)
    assert np.array_equal(y[0], q[:, 7] + res[0].astype(np.float64))
    assert np.array_equal(y[1], q[:, 40] + res[1].astype(np.float64))


def test_rmsnorm_quantize_closed_forms():
    """O9: a constant row c has r = 1/sqrt(c^2 + eps) (0.5 exactly for c = 2,
    eps = 0); the row (3, 4, 0, ...) of K = 32 has mean square 25/32, so xhat =
    (3r, 4r, 0, ...), amax = 4r and the codes are round(95.25) = 95 and 127
    whatever r rounds to; doubling x halves r and leaves xhat and the codes
    unchanged (eps = 0); the mean of squares matches exact rationals."""
    from fractions import Fraction
    K = 64
    r, xh, q, d, _ = oracle.rmsnorm_quantize_act(np.full((1, K), 2.0, np.float32), np.ones(K, np.float32), 0.0)
    assert r[0] == 0.5 and np.all(xh == 1.0) and np.all(q == 127)
    x = np.zeros((1, 32), np.float32)
    x[0, 0], x[0, 1] = 3.0, 4.0
    r, xh, q, d, _ = oracle.rmsnorm_quantize_act(x, np.ones(32, np.float32), 0.0)
    assert abs(r[0] - (32 / 25) ** 0.5) < 1e-15
    assert q[0, 0] == 95 and q[0, 1] == 127 and np.all(q[0, 2:] == 0)
    rng = np.random.default_rng(8)
    x = rng.standard_normal((3, 96)).astype(np.float32)
    g = (1 + 0.1 * rng.standard_normal(96)).astype(np.float32)
    r1, xh1, q1, d1, _ = oracle.rmsnorm_quantize_act(x, g, 0.0)
    r2, xh2, q2, d2, _ = oracle.rmsnorm_quantize_act(2 * x, g, 0.0)
    assert np.allclose(r2, r1 / 2, rtol=1e-15, atol=0)
    assert np.array_equal(xh1, xh2) and np.array_equal(q1, q2) and np.array_equal(d1, d2)
    for n in range(3):
        ms = sum(Fraction(float(v)) ** 2 for v in x[n]) / 96
        assert abs(1.0 / r1[n] ** 2 - float(ms)) <= 1e-14 * float(ms)
    # gamma = 1 and r = 1 reduce O9 to the plain quantiser O5
    _, _, q3, d3, _ = oracle.rmsnorm_quantize_act(x, np.ones(96, np.float32), 0.0, r=np.ones(3, np.float32))
    q4, d4, _ = oracle.quantize_act(x)
    assert np.array_equal(q3, q4) and np.array_equal(d3, d4)


def test_int_dots_closed_forms():
    K = 64
    qw = np.full((2, K), 127, np.int8)
    qw[1, ::2] = -127
    g = q8gen.assemble_gguf(qw, np.full((2, 2), 0x3C00, np.uint16))
    xq = np.full((1, K), 127, np.int8)
    xd = np.full((1, 2), 0x3C00, np.uint16)
    dots, y, _ = oracle.q8q8(g, xq, xd, 2, K)
    assert dots[0, 0].tolist() == [516128, 516128]
    assert dots[0, 1].tolist() == [0, 0]
    assert y[0].tolist() == [2 * 516128.0, 0.0]


# --------------------------------------------------------------------------
# P8: router
# --------------------------------------------------------------------------

def test_router_closed_forms():
    E = 60
    idx, w = oracle.route(np.zeros((1, E), np.float32), 4)
    assert idx[0].tolist() == [0, 1, 2, 3]
    assert np.allclose(w[0], 1 / 60, rtol=1e-15, atol=0)
    ramp = np.arange(E, dtype=np.float32).reshape(1, E)
    idx, w = oracle.route(ramp, 4)
    assert idx[0].tolist() == [59, 58, 57, 56]
    # softmax of a ramp: p_e = e^e / sum_j e^j, a geometric series
    z = sum(math.exp(j - 59) for j in range(E))
    assert np.allclose(w[0], [math.exp(e - 59) / z for e in (59, 58, 57, 56)], rtol=1e-14)
    # ties: equal top values resolve to the lower index, in order
    l = np.full((1, E), -1.0, np.float32)
    l[0, [7, 3, 40, 12, 5]] = 2.0
    idx, _ = oracle.route(l, 4)
    assert idx[0].tolist() == [3, 5, 7, 12]
    # probabilities of all E experts sum to one: with k = E
    lg = q8gen.logits(3, 5, E)
    idx, w = oracle.route(lg, E)
    assert np.allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    assert all(sorted(r) == list(range(E)) for r in idx.tolist())
    # descending order of the logits
    for t in range(5):
        assert np.all(np.diff(lg[t, idx[t]]) <= 0)
    # renormalised weights sum to one over the picks
    _, wr = oracle.route(lg, 4, renormalize=True)
    assert np.allclose(wr.sum(axis=1), 1.0, rtol=0, atol=1e-14)


# --------------------------------------------------------------------------
# P9: SwiGLU closed forms
# --------------------------------------------------------------------------

def _unit_matrix(q_rows):
    q = np.array(q_rows, np.int8)
    return q8gen.assemble_gguf(q, np.full((q.shape[0], q.shape[1] // 32), 0x3C00, np.uint16))


def test_swiglu_closed_forms():
    K = 32
    # gate row picks x0, up row picks x1
    qg = np.zeros((1, K), np.int8); qg[0, 0] = 1
    qu = np.zeros((1, K), np.int8); qu[0, 1] = 1
    g8 = _unit_matrix(np.concatenate([qg, qu]))
    ln3 = np.float32(math.log(3.0))
    x = np.zeros((3, K), np.float32)
    x[0, :2] = [0.0, 5.0]     # g = 0            -> h = 0
    x[1, :2] = [ln3, 4.0]     # sigmoid(ln 3) = 3/4 -> h = 0.75 * ln3 * 4
    x[2, :2] = [-ln3, 4.0]    # silu(-g) = silu(g) - g
    out = oracle.gate_up_swiglu(g8, x, 1, K)
    h = out["h"][:, 0]
    assert h[0] == 0.0
    g = float(ln3)
    assert abs(h[1] - 3.0 * g) <= 4 * 1e-7  # sigmoid(fp32(ln3)) = 3/4 + O(1e-8)
    assert abs(h[2] - (h[1] - 4 * g)) <= 1e-12
    # large gate: silu(g) ~ g;  very negative gate: ~ 0
    x2 = np.zeros((2, K), np.float32)
    x2[0, :2] = [40.0, 1.5]
    x2[1, :2] = [-40.0, 1.5]
    h2 = oracle.gate_up_swiglu(g8, x2, 1, K)["h"][:, 0]
    assert abs(h2[0] - 60.0) <= 60.0 * 1e-15
    assert abs(h2[1]) <= 1e-15


# --------------------------------------------------------------------------
# P10: the MoE block reduces to the dense SwiGLU MLP
# --------------------------------------------------------------------------

def test_moe_reduces_to_dense():
    H, I = 64, 96
    gu, _ = q8gen.q8_matrix(41, 2 * I, H)
    dn, _ = q8gen.q8_matrix(42, H, I)
    x = q8gen.activations(43, 2, H)
    idx = np.zeros((2, 1), np.int32)
    w = np.ones((2, 1), np.float64)
    y, bound, slot = oracle.moe(gu, dn, None, None, idx, w, x, H, I, 0)
    # dense MLP: h = SwiGLU(gate_up x), then down h, with h exact in fp64
    h = oracle.gate_up_swiglu(gu, x, I, H)["h"]
    q, dbits = q8gen.split_gguf(dn, H, I)
    wd = q.astype(np.float64) * np.repeat(dbits.view(np.float16).astype(np.float64), 32, axis=1)
    dense = h @ wd.T
    assert np.allclose(y, dense, rtol=1e-12, atol=1e-12 * np.abs(h).max())
    assert np.array_equal(slot[:, 0], y)
    assert np.all(bound > 0)
    # a shared expert is added with weight one
    y2, _, _ = oracle.moe(gu, dn, gu, dn, idx, w, x, H, I, I)
    assert np.allclose(y2, 2 * y, rtol=1e-12, atol=1e-12 * np.abs(y).max())
    # two slots on the same expert with weights a, b scale its output by a + b
    idx2 = np.zeros((2, 2), np.int32)
    w2 = np.array([[0.25, 0.5], [0.125, 1.0]])
    gu2 = np.concatenate([gu, gu])  # E = 2 identical experts
    dn2 = np.concatenate([dn, dn])
    y3, _, _ = oracle.moe(gu2, dn2, None, None, idx2 + np.array([[0, 1]]), w2, x, H, I, 0)
    assert np.allclose(y3, y * w2.sum(axis=1)[:, None], rtol=1e-12, atol=1e-12 * np.abs(y).max())


def _dense_mlp(gu_bytes, dn_bytes, x_row, H, I):
    """One expert's SwiGLU MLP on one token: h from O2 on that expert's own
    gate_up bytes, then its down matrix decoded from its GGUF bytes by numpy
    and applied in fp64."""
    h = oracle.gate_up_swiglu(gu_bytes, x_row[None, :], I, H)["h"][0]
    q, dbits = q8gen.split_gguf(dn_bytes, H, I)
    wd = q.astype(np.float64) * np.repeat(dbits.view(np.float16).astype(np.float64), 32, axis=1)
    return wd @ h


def test_moe_distinct_experts_match_dense_mlps():
    """O4 with several *different* experts: every token's output is the
    weighted sum of the dense MLPs of exactly the experts its idx row names,
    in any slot position, plus the shared expert with weight one (the router +
    top-k expert + shared-expert FFN block of the GPULlama3.java Qwen1.5-MoE
    pull request, PR summary).  Each expert's MLP is computed from its own byte
    slice of the stacked buffers, so reading the wrong expert (a fixed index,
    the slot number in place of idx, a wrong stride) changes the result."""
    H, I, Is, E = 64, 96, 64, 5
    gu_list, dn_list = [], []
    for e in range(E):
        gu_list.append(q8gen.q8_matrix(300 + e, 2 * I, H)[0])
        dn_list.append(q8gen.q8_matrix(400 + e, H, I)[0])
    sgu = q8gen.q8_matrix(500, 2 * Is, H)[0]
    sdn = q8gen.q8_matrix(501, H, Is)[0]
    gu_all, dn_all = np.concatenate(gu_list), np.concatenate(dn_list)
    x = q8gen.activations(502, 4, H)
    # distinct experts in different slot positions, one token reusing another's
    # expert in the other slot, unequal weights
    idx = np.array([[3, 1, 4], [0, 2, 3], [4, 3, 1], [2, 0, 4]], np.int32)
    w = np.array([[0.5, 0.25, 0.125], [0.375, 0.0625, 0.3125], [0.2, 0.7, 0.1], [0.9, 0.05, 0.05]])
    y, bound, slot = oracle.moe(gu_all, dn_all, None, None, idx, w, x, H, I, 0)
    ys, _, _ = oracle.moe(gu_all, dn_all, sgu, sdn, idx, w, x, H, I, Is)
    for t in range(idx.shape[0]):
        want = np.zeros(H)
        for s in range(idx.shape[1]):
            e = int(idx[t, s])
            o = _dense_mlp(gu_list[e], dn_list[e], x[t], H, I)
            assert np.allclose(slot[t, s], o, rtol=1e-12, atol=1e-12 * np.abs(o).max())
            want += w[t, s] * o
        assert np.allclose(y[t], want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
        sh = _dense_mlp(sgu, sdn, x[t], H, Is)
        assert np.allclose(ys[t], want + sh, rtol=1e-12, atol=1e-12 * np.abs(want + sh).max())
    # the experts really differ: swapping two picks of a token changes its output
    idx2 = idx.copy()
    idx2[0, [0, 1]] = idx2[0, [1, 0]]
    y2, _, _ = oracle.moe(gu_all, dn_all, None, None, idx2, w, x, H, I, 0)
    assert np.abs(y2[0] - y[0]).max() > 1e-3 * np.abs(y[0]).max()
    assert np.array_equal(y2[1:], y[1:])
    assert np.all(bound > 0)
