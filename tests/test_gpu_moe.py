"""GPU parity of the grouped MoE GEMV (S6) against the CPU oracle.

The oracle computes the MoE block in fp64 (router + top-k experts + shared
expert) and a per-output error bound carried from the 1e-5 * sum|w x| GEMV
tolerance through SwiGLU and the down projection.  The GPU block is fed the
GPU router's indices (checked equal to the oracle's) and weights (the oracle
uses the same weights, so the bound needs no weight-error term)."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import q8gen
from q8_test_utils import assert_within, dev, dev_bytes, torch

pytestmark = pytest.mark.gpu


def q8():
    import q8_block_quantized_02_b200 as m
    return m


def pack_stack(gguf_all: np.ndarray, E: int, M: int, K: int):
    """Pack E consecutive GGUF matrices [M][K] into E consecutive packed ones."""
    t = torch()
    m = q8()
    one = m.q8_packed_bytes(M, K)
    src = dev_bytes(gguf_all)
    out = t.empty(E * one, dtype=t.uint8, device="cuda")
    g_one = M * (K // 32) * 34
    for e in range(E):
        m.q8_pack_weights(src[e * g_one:(e + 1) * g_one], M, K, out[e * one:(e + 1) * one])
    return out


class MoeCase:
    def __init__(self, E, H, I, Is, seed=0):
        self.E, self.H, self.I, self.Is = E, H, I, Is
        gu = np.concatenate([q8gen.q8_matrix(seed * 1000 + e, 2 * I, H)[0] for e in range(E)])
        dn = np.concatenate([q8gen.q8_matrix(seed * 1000 + 500 + e, H, I)[0] for e in range(E)])
        self.gu, self.dn = gu, dn
        self.p_gu = pack_stack(gu, E, 2 * I, H)
        self.p_dn = pack_stack(dn, E, H, I)
        if Is:
            self.sgu = q8gen.q8_matrix(seed * 1000 + 900, 2 * Is, H)[0]
            self.sdn = q8gen.q8_matrix(seed * 1000 + 901, H, Is)[0]
            self.p_sgu = pack_stack(self.sgu, 1, 2 * Is, H)
            self.p_sdn = pack_stack(self.sdn, 1, H, Is)
        else:
            self.sgu = self.sdn = self.p_sgu = self.p_sdn = None

    def run(self, x, k, renorm=False, logits=None, seed=7):
        t = torch()
        m = q8()
        T = x.shape[0]
        lg = logits if logits is not None else q8gen.logits(seed, T, self.E)
        idx = t.empty((T, k), dtype=t.int32, device="cuda")
        w = t.empty((T, k), dtype=t.float32, device="cuda")
        m.q8_moe_route(dev(lg), T, self.E, k, renorm, idx, w)
        ws_bytes = m.q8_moe_workspace_bytes(T, self.E, k, self.H, self.I, self.Is)
        ws = t.full((ws_bytes // 4,), float("nan"), dtype=t.float32, device="cuda")
        m.q8_moe_workspace_init(ws, ws_bytes)
        y = t.full((T, self.H), float("nan"), dtype=t.float32, device="cuda")
        m.q8_moe_gemv(self.p_gu, self.p_dn, self.p_sgu, self.p_sdn, idx, w, dev(x), y, T, self.E, k,
                      self.H, self.I, self.Is, ws, ws_bytes)
        return lg, idx.cpu().numpy(), w.cpu().numpy(), y.cpu().numpy()

    def gemv_raw(self, idx, w, x, ws, ws_bytes):
        """One q8_moe_gemv call with the given (device) idx and w on a given workspace."""
        t = torch()
        T, k = idx.shape
        y = t.full((T, self.H), float("nan"), dtype=t.float32, device="cuda")
        q8().q8_moe_gemv(self.p_gu, self.p_dn, self.p_sgu, self.p_sdn, idx, w, dev(x), y, T, self.E, k,
                         self.H, self.I, self.Is, ws, ws_bytes)
        return y.cpu().numpy()

    def check(self, x, k, renorm=False, logits=None, seed=7, what=""):
        lg, idx, w, y = self.run(x, k, renorm, logits, seed)
        idx_ref, _ = oracle.route(lg, k, renorm)
        assert np.array_equal(idx, idx_ref), "router indices differ"
        y_ref, bound, _ = oracle.moe(self.gu, self.dn, self.sgu, self.sdn, idx, w.astype(np.float64),
                                     x, self.H, self.I, self.Is, threads=oracle.max_threads())
        return assert_within(y, y_ref, bound, what)


@pytest.mark.parametrize("E,H,I,Is", [(8, 64, 96, 128), (12, 96, 64, 0), (5, 32, 32, 32)])
@pytest.mark.parametrize("T,k", [(1, 1), (2, 2), (3, 2), (8, 4), (16, 3)])
def test_moe_small_matches_oracle(E, H, I, Is, T, k):
    case = MoeCase(E, H, I, Is, seed=E + H)
    x = q8gen.activations(T * 31 + E, T, H)
    case.check(x, k, what=f"moe E={E} H={H} I={I} Is={Is} T={T} k={k}")


def test_moe_renormalized_and_shared_picks():
    case = MoeCase(6, 64, 64, 64, seed=3)
    x = q8gen.activations(5, 8, 64)
    case.check(x, 4, renorm=True, what="renormalised")
    # every token picks the same experts: one expert serves all tokens
    lg = np.tile(np.arange(6, dtype=np.float32), (8, 1))
    case.check(x, 2, logits=lg, what="shared picks")


@pytest.fixture(scope="module")
def qwen_moe():
    """Qwen1.5-MoE-A2.7B shapes: hidden 2048, 60 experts of intermediate 1408,
    shared expert of intermediate 5632."""
    return MoeCase(60, 2048, 1408, 5632, seed=11)


@pytest.mark.parametrize("T", [1, 8])
def test_moe_qwen_shapes(qwen_moe, T):
    x = q8gen.activations(61, T, 2048)
    ratio = qwen_moe.check(x, 4, seed=61 + T, what=f"qwen moe T={T}")
    assert ratio < 1.0


def test_moe_deterministic(qwen_moe):
    x = q8gen.activations(62, 8, 2048)
    _, _, _, y1 = qwen_moe.run(x, 4, seed=9)
    _, _, _, y2 = qwen_moe.run(x, 4, seed=9)
    assert np.array_equal(y1, y2)


def test_moe_workspace_reused_across_calls():
    """Calls of different token counts and routings in a row on one
    workspace, zero-filled once: the counters each call leaves behind must
    let the next one run correctly, and end zero."""
    t = torch()
    m = q8()
    case = MoeCase(10, 96, 64, 96, seed=4)
    k = 3
    ws_bytes = max(m.q8_moe_workspace_bytes(T, case.E, k, case.H, case.I, case.Is) for T in (1, 5, 16))
    ws = t.empty(ws_bytes, dtype=t.uint8, device="cuda")
    m.q8_moe_workspace_init(ws, ws_bytes)
    for call, T in enumerate((5, 1, 16, 5)):
        x = q8gen.activations(70 + call, T, case.H)
        lg = q8gen.logits(80 + call, T, case.E)
        idx = t.empty((T, k), dtype=t.int32, device="cuda")
        w = t.empty((T, k), dtype=t.float32, device="cuda")
        m.q8_moe_route(dev(lg), T, case.E, k, 0, idx, w)
        y = case.gemv_raw(idx, w, x, ws, ws_bytes)
        y_ref, bound, _ = oracle.moe(case.gu, case.dn, case.sgu, case.sdn, idx.cpu().numpy(),
                                     w.cpu().numpy().astype(np.float64), x, case.H, case.I, case.Is)
        assert_within(y, y_ref, bound, f"call {call} (T={T})")
    assert m.q8_read_device_error() == (0, 0)
    # the counters come first in the workspace (2 + 128 per-segment words, then
    # one per 8 output rows); every call leaves them zero
    head = ws[:4 * (2 + 128 + case.H // 8)].cpu().numpy()
    assert not head.any()


def test_moe_rejected_picks():
    """A pick outside [0, E) and a token's second pick of the same expert add
    nothing and set bit 4 of the device error word; the other picks and the
    shared expert still give the oracle's values."""
    t = torch()
    m = q8()
    case = MoeCase(6, 64, 64, 64, seed=5)
    T, k = 4, 3
    x = q8gen.activations(90, T, case.H)
    idx = np.array([[0, 7, 2], [3, 3, 1], [-1, 5, 4], [2, 4, 0]], np.int32)
    wts = np.array([[0.5, 0.25, 0.25], [0.4, 0.3, 0.3], [0.2, 0.3, 0.5], [0.1, 0.6, 0.3]], np.float32)
    ws_bytes = m.q8_moe_workspace_bytes(T, case.E, k, case.H, case.I, case.Is)
    ws = t.empty(ws_bytes, dtype=t.uint8, device="cuda")
    m.q8_moe_workspace_init(ws, ws_bytes)
    m.q8_read_device_error()
    y = case.gemv_raw(t.from_numpy(idx).cuda(), t.from_numpy(wts).cuda(), x, ws, ws_bytes)
    st, word = m.q8_read_device_error()
    assert word == 4
    # the oracle with the rejected picks given weight zero (on a valid expert)
    keep = np.ones_like(wts, dtype=bool)
    keep[0, 1] = keep[1, 1] = keep[2, 0] = False
    idx_ok = np.where(keep, idx, 0)
    w_ok = np.where(keep, wts, 0.0).astype(np.float64)
    y_ref, bound, _ = oracle.moe(case.gu, case.dn, case.sgu, case.sdn, idx_ok, w_ok, x, case.H, case.I,
                                 case.Is)
    assert_within(y, y_ref, bound, "rejected picks")


def test_moe_validation():
    m = q8()
    t = torch()
    case = MoeCase(4, 32, 32, 32, seed=1)
    T, k = 2, 2
    idx = t.tensor([[0, 1], [2, 1]], dtype=t.int32, device="cuda")  # distinct picks per token
    w = t.ones((T, k), dtype=t.float32, device="cuda")
    x = dev(q8gen.activations(1, T, 32))
    y = t.empty((T, 32), dtype=t.float32, device="cuda")
    need = m.q8_moe_workspace_bytes(T, 4, k, 32, 32, 32)
    ws = t.empty((need // 4,), dtype=t.float32, device="cuda")
    m.q8_moe_workspace_init(ws, need)

    def status(*a):
        with pytest.raises(m.Q8Error) as e:
            m.q8_moe_gemv(*a)
        return e.value.status

    base = [case.p_gu, case.p_dn, case.p_sgu, case.p_sdn, idx, w, x, y, T, 4, k, 32, 32, 32, ws, need]
    bad = list(base); bad[15] = need - 4
    assert status(*bad) == 2                      # workspace too small
    bad = list(base); bad[2] = None
    assert status(*bad) == 1                      # half a shared expert
    bad = list(base); bad[8] = 17
    assert status(*bad) == 5                      # too many tokens
    bad = list(base); bad[11] = 48
    assert status(*bad) == 2                      # H % 32
    m.q8_moe_gemv(*base)
    assert m.q8_read_device_error() == (0, 0)
