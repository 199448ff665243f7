"""GPU test of the failure-detection protocol: a bounded wait that runs out.

Every barrier wait in the library's kernels is bounded; a wait that runs past
its limit sets a bit in the sticky device error word, raises its CTA's abort
flag so the CTA's other warps leave their waits, and the kernel returns.  The
test aid q8_test_wait_timeout runs that same wait code on a barrier that
nothing completes, with a limit of a few milliseconds: no fault, no trap, no
hang.  The host then reads the error word, and the context must still run a
product correctly."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from q8_test_utils import TOL_REL, assert_within, gemv, matrix, pack, torch

pytestmark = pytest.mark.gpu


def q8():
    import q8_block_quantized_02_b200 as m
    return m


def test_wait_runs_out_and_is_reported():
    t = torch()
    m = q8()
    assert m.q8_read_device_error() == (0, 0)
    out = t.full((2,), -1, dtype=t.int32, device="cuda")
    m.q8_test_wait_timeout(5000, out)
    st, word = m.q8_read_device_error()
    assert st == 7 and word & 1, (st, word)     # Q8_ERR_DEVICE_TIMEOUT, timeout bit
    assert out.cpu().tolist() == [0, 1]         # no warp's wait succeeded; abort raised
    assert m.q8_read_device_error() == (0, 0)   # reading cleared the word
    # the context is intact: a product right after is correct
    M, K = 1152, 896
    g, x = matrix(3, M, K, 1)
    y = gemv(pack(g, M, K), x, M, K)
    y_ref, y_abs = oracle.gemv(g, x, M, K)
    assert_within(y, y_ref, TOL_REL * y_abs, "gemv after a timed-out wait")
    assert m.q8_read_device_error() == (0, 0)


def test_wait_timeout_rejects_bad_limits():
    t = torch()
    m = q8()
    out = t.empty((2,), dtype=t.int32, device="cuda")
    for limit in (0, 2_000_000):
        with pytest.raises(m.Q8Error) as e:
            m.q8_test_wait_timeout(limit, out)
        assert e.value.status == 5
    with pytest.raises(m.Q8Error) as e:
        m.q8_test_wait_timeout(1000, 0)
    assert e.value.status == 1
