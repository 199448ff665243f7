"""Helpers shared by the GPU tests: upload, pack, tolerance checks.

Inputs come from ``q8gen`` (seeded, synthetic), expected values from
``oracle`` (fp64 CPU); the CUDA path is called only through the C ABI via the
package's binding."""
from __future__ import annotations

import numpy as np

import q8gen

TOL_REL = 1e-5  # |y - y_ref| <= 1e-5 * sum_k |w_k x_k|


def torch():
    import torch as _t
    return _t


def dev_bytes(arr: np.ndarray):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(arr).view(np.uint8).reshape(-1).copy()).cuda()


def dev(arr: np.ndarray):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(arr).copy()).cuda()


def pack(gguf: np.ndarray, M: int, K: int):
    """Upload GGUF bytes and pack them on the GPU; returns the packed tensor."""
    import q8_block_quantized_02_b200 as q8
    t = torch()
    g = dev_bytes(gguf)
    packed = t.empty(q8.q8_packed_bytes(M, K), dtype=t.uint8, device="cuda")
    q8.q8_pack_weights(g, M, K, packed)
    return packed


def gemv(packed, x: np.ndarray, M: int, K: int, split: bool = False):
    """q8_gemv (or, with split, q8_gemv_split) on x; returns y [N][M]."""
    import q8_block_quantized_02_b200 as q8
    t = torch()
    xd = dev(x.astype(np.float32))
    N = x.shape[0]
    y = t.full((N, M), float("nan"), dtype=t.float32, device="cuda")
    (q8.q8_gemv_split if split else q8.q8_gemv)(packed, xd, y, M, K, N)
    return y.cpu().numpy()


def gate_up(packed, x: np.ndarray, I: int, K: int, split: bool = False):
    """q8_gate_up_swiglu (or its split variant) on x; returns h [N][I]."""
    import q8_block_quantized_02_b200 as q8
    t = torch()
    xd = dev(x.astype(np.float32))
    N = x.shape[0]
    h = t.full((N, I), float("nan"), dtype=t.float32, device="cuda")
    (q8.q8_gate_up_swiglu_split if split else q8.q8_gate_up_swiglu)(packed, xd, h, I, K, N)
    return h.cpu().numpy()


def assert_within(y: np.ndarray, y_ref: np.ndarray, bound: np.ndarray, what: str = ""):
    y = y.astype(np.float64)
    assert np.all(np.isfinite(y)), f"{what}: non-finite outputs"
    err = np.abs(y - y_ref)
    bad = err > bound
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside tolerance; first at "
                             f"{tuple(i)}: got {y[tuple(i)]!r} want {y_ref[tuple(i)]!r} "
                             f"err {err[tuple(i)]:.3e} bound {bound[tuple(i)]:.3e}")
    return float((err / np.maximum(bound, 1e-300)).max()) if err.size else 0.0


def swiglu_bound(ref: dict) -> np.ndarray:
    """Error bound on h carried from the GEMV tolerance on g and u
    (|silu'| <= 1.1), plus a few ulps for the fp32 SiLU itself."""
    g, u, h = ref["g"], ref["u"], ref["h"]
    tg, tu = TOL_REL * ref["g_abs"], TOL_REL * ref["u_abs"]
    silu = g / (1.0 + np.exp(-g))
    return 1.1 * tg * np.abs(u) + np.abs(silu) * tu + 1.1 * tg * tu + 4 * 2.0 ** -23 * np.abs(h)


def rows_subset(gguf: np.ndarray, M: int, K: int, rows: np.ndarray) -> np.ndarray:
    """GGUF bytes of the given rows only (rows are contiguous runs of K/32 blocks)."""
    b = np.ascontiguousarray(gguf).reshape(M, (K // 32) * 34)
    return np.ascontiguousarray(b[rows]).reshape(-1)


def matrix(seed: int, M: int, K: int, N: int | None = None):
    return q8gen.q8_matrix(seed, M, K, N)


def pack_q6k_reference(blocks, M, K):
    """The packed layout as include/q8.h states it, written with numpy: unit
    (t, b) of 6720 bytes; row i of tile t at byte 208 i holds raw bytes 0..207
    of block b of matrix row 32t + i, bytes 6656 + 2i, + 1 its d; rows past M
    zero."""
    SB = K // 256
    T = -(-M // 32)
    raw = np.zeros((T * 32, SB, 210), np.uint8)
    raw[:M] = blocks.reshape(M, SB, 210)
    raw = raw.reshape(T, 32, SB, 210).transpose(0, 2, 1, 3)  # [t][b][i][210]
    out = np.zeros((T, SB, 6720), np.uint8)
    out[:, :, :6656] = raw[:, :, :, :208].reshape(T, SB, 6656)
    out[:, :, 6656:] = raw[:, :, :, 208:].reshape(T, SB, 64)
    return out.reshape(-1)
