"""GPU test of q8_moe_gemv_noalloc, the MoE entry point that takes no
workspace (for callers that cannot allocate device memory when they call).

It is checked against the workspace-taking q8_moe_gemv, on two calls in a row
with different inputs (the built-in scratch keeps the previous call's
contents), and both against the fp64 oracle's error bound.  This file is
named so that pytest collects it after every other test; it also passes when
run alone in a fresh process (its first call sets up the scratch address)."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import q8gen

pytestmark = pytest.mark.gpu


def _torch():
    import torch
    return torch


def _pack_stack(gguf_all, E, M, K):
    import q8_block_quantized_02_b200 as q8
    t = _torch()
    one = q8.q8_packed_bytes(M, K)
    src = t.from_numpy(gguf_all.copy()).cuda()
    out = t.empty(E * one, dtype=t.uint8, device="cuda")
    g_one = M * (K // 32) * 34
    for e in range(E):
        q8.q8_pack_weights(src[e * g_one:(e + 1) * g_one], M, K, out[e * one:(e + 1) * one])
    return out


def test_noalloc_matches_workspace_entry_point():
    import q8_block_quantized_02_b200 as q8
    t = _torch()
    E, H, I, Is, k = 8, 128, 96, 160, 2
    gu = np.concatenate([q8gen.q8_matrix(100 + e, 2 * I, H)[0] for e in range(E)])
    dn = np.concatenate([q8gen.q8_matrix(200 + e, H, I)[0] for e in range(E)])
    sgu = q8gen.q8_matrix(300, 2 * Is, H)[0]
    sdn = q8gen.q8_matrix(301, H, Is)[0]
    p_gu, p_dn = _pack_stack(gu, E, 2 * I, H), _pack_stack(dn, E, H, I)
    p_sgu, p_sdn = _pack_stack(sgu, 1, 2 * Is, H), _pack_stack(sdn, 1, H, Is)

    for call, T in enumerate((5, 3)):  # two calls in a row, different inputs
        x = q8gen.activations(400 + call, T, H)
        lg = q8gen.logits(500 + call, T, E)
        idx = t.empty((T, k), dtype=t.int32, device="cuda")
        w = t.empty((T, k), dtype=t.float32, device="cuda")
        q8.q8_moe_route(t.from_numpy(lg).cuda(), T, E, k, 0, idx, w)
        xd = t.from_numpy(x).cuda()

        y_noalloc = t.full((T, H), float("nan"), dtype=t.float32, device="cuda")
        q8.q8_moe_gemv_noalloc(p_gu, p_dn, p_sgu, p_sdn, idx, w, xd, y_noalloc, T, E, k, H, I, Is)

        ws_bytes = q8.q8_moe_workspace_bytes(T, E, k, H, I, Is)
        ws = t.empty(ws_bytes, dtype=t.uint8, device="cuda")
        q8.q8_moe_workspace_init(ws, ws_bytes)
        y_ws = t.full((T, H), float("nan"), dtype=t.float32, device="cuda")
        q8.q8_moe_gemv(p_gu, p_dn, p_sgu, p_sdn, idx, w, xd, y_ws, T, E, k, H, I, Is, ws, ws_bytes)

        a = y_noalloc.cpu().numpy().astype(np.float64)
        b = y_ws.cpu().numpy().astype(np.float64)
        y_ref, bound, _ = oracle.moe(gu, dn, sgu, sdn, idx.cpu().numpy(),
                                     w.cpu().numpy().astype(np.float64), x, H, I, Is)
        assert np.all(np.isfinite(a))
        assert np.all(np.abs(a - b) <= bound), f"call {call}: no-alloc differs from the workspace path"
        assert np.all(np.abs(a - y_ref) <= bound), f"call {call}: no-alloc outside the oracle bound"
    st, word = q8.q8_read_device_error()
    assert st == 0 and word == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import q8_block_quantized_02_b200 as q8
    # 16 tokens x 8 slots x 8192 floats of routed h alone fill the 4 MiB scratch
    T, E, k, H, I, Is = 16, 64, 8, 2048, 8192, 32
    assert q8.q8_moe_workspace_bytes(T, E, k, H, I, Is) > 4 << 20
    with pytest.raises(q8.Q8Error) as e:
        q8.q8_moe_gemv_noalloc(16, 16, 16, 16, 16, 16, 16, 16, T, E, k, H, I, Is)
    assert e.value.status == 5
