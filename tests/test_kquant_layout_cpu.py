"""CPU check of the packed Q6_K layout that the GPU pack test compares
against: the numpy re-statement (q8_test_utils.pack_q6k_reference) against a
per-byte loop written from the layout's definition in include/q8.h, on a
ragged tile and several blocks per row."""
from __future__ import annotations

import numpy as np

import q8gen
from q8_test_utils import pack_q6k_reference


def _pack_by_bytes(blocks: np.ndarray, M: int, K: int) -> np.ndarray:
    """unit (t, b) at byte (t * SB + b) * 6720; row i of tile t at byte 208 i
    of the unit holds bytes 0..207 of raw block (32 t + i, b); bytes
    6656 + 2 i and 6657 + 2 i hold raw bytes 208, 209 (its d); rows past M are
    zero."""
    SB = K // 256
    T = (M + 31) // 32
    out = np.zeros(T * SB * 6720, np.uint8)
    for t in range(T):
        for b in range(SB):
            base = (t * SB + b) * 6720
            for i in range(32):
                row = 32 * t + i
                if row >= M:
                    continue
                src = (row * SB + b) * 210
                for o in range(208):
                    out[base + 208 * i + o] = blocks[src + o]
                out[base + 6656 + 2 * i] = blocks[src + 208]
                out[base + 6657 + 2 * i] = blocks[src + 209]
    return out


def test_q6k_packed_layout_matches_its_definition():
    M, K = 45, 768  # two tiles (the second ragged), three blocks a row
    blocks = q8gen.kquant_matrix("q6_k", 5, M, K)
    ref = _pack_by_bytes(blocks, M, K)
    assert ref.size == 2 * 3 * 6720
    assert np.array_equal(pack_q6k_reference(blocks, M, K), ref)
    # the padding rows of the last tile are zero, and every raw byte appears
    assert ref.sum(dtype=np.int64) == blocks.sum(dtype=np.int64)
