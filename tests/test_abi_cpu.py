"""CPU-only checks of the C-ABI library: it builds for sm_100a, loads, exports
every symbol include/q8.h declares, and its pure host queries answer as
documented.  No compute call is made (there is no GPU here)."""
from __future__ import annotations

import ctypes
import os
import re
import shutil

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "q8.h")


def _header_text() -> str:
    return re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)


def _inline_helpers() -> list[str]:
    """static inline functions the header defines (decoders; not exported)."""
    return sorted(set(re.findall(r"static\s+inline\s+[\w\s\*]*?\b(q8\w*)\s*\(", _header_text())))


def _declared_functions() -> list[str]:
    """Entry points the library must export: every q8* function the header
    names, less its static inline helpers."""
    names = set(re.findall(r"\b(q8\w*)\s*\(", _header_text()))
    return sorted(names - set(_inline_helpers()))


@pytest.fixture(scope="module")
def lib():
    if shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"):
        pytest.skip("nvcc not available")
    from q8_block_quantized_02_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("q8_pack_weights", "q8_gemv", "q8_gate_up_swiglu", "q8_moe_route",
                     "q8_moe_gemv", "q8_quantize_act", "q8q8_gemv", "q8q8_block_dots",
                     "q8_packed_bytes", "q8_moe_workspace_bytes", "q8_moe_workspace_init",
                     "q8_unpack_weights"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, f"not exported: {missing}"


def test_binding_covers_the_header():
    import q8_block_quantized_02_b200 as q8
    for n in _declared_functions() + _inline_helpers():
        assert hasattr(q8, n), f"python binding lacks {n}"


def test_header_compiles_as_c_and_cpp(tmp_path):
    """include/q8.h is a C ABI: a translation unit using it compiles as strict
    C99 and as C++, and a C program built on its inline key decoders gives
    back what a key was made from."""
    import subprocess
    if shutil.which("gcc") is None or shutil.which("g++") is None:
        pytest.skip("gcc / g++ not available")
    inc = os.path.join(ROOT, "include")
    uses = tmp_path / "uses_entry_points.c"
    uses.write_text(
        '#include "q8.h"\n'
        "q8_status call_gemv(const void *w, const float *x, float *y) {\n"
        "  return q8_gemv(w, x, y, 8, 32, 1, (q8_stream_t)0);\n}\n")
    for cmd in (["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-c"],
                ["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-x", "c++", "-c"]):
        subprocess.run(cmd + ["-I", inc, str(uses), "-o", str(tmp_path / "uses.o")], check=True)
    prog = tmp_path / "decode_key.c"
    prog.write_text(
        '#include "q8.h"\n#include <stdio.h>\n'
        "int main(void) {\n"
        "  uint64_t k = ((uint64_t)(0x80000000u | 0x3FC00000u) << 32) | (0xFFFFFFFFu - 7u);\n"
        '  printf("%d %g\\n", q8_argmax_index(k), (double)q8_argmax_value(k));\n'
        "  return 0;\n}\n")
    exe = tmp_path / "decode_key"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", inc, str(prog), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    assert out == ["7", "1.5"]


def test_argmax_key_decoders():
    """The header's key layout: order-preserving float bits high, 0xFFFFFFFF -
    index low; the binding's decoders invert it for every sign and size."""
    import numpy as np
    import q8_block_quantized_02_b200 as q8
    assert "q8_argmax_index" in _inline_helpers() and "q8_argmax_value" in _inline_helpers()
    vals = np.array([0.0, 1.5, -1.5, 3.4e38, -3.4e38, 1e-45, -1e-45, 7.0], np.float32)
    idx = np.array([0, 1, 151935, 7, 2**30, 12, 13, 5], np.int64)
    u = vals.view(np.uint32).astype(np.uint64)
    ordered = np.where(u & 0x80000000, ~u & 0xFFFFFFFF, u | 0x80000000)
    keys = (ordered << np.uint64(32)) | (np.uint64(0xFFFFFFFF) - idx.astype(np.uint64))
    assert np.array_equal(q8.q8_argmax_index(keys), idx)
    assert np.array_equal(q8.q8_argmax_value(keys).view(np.uint32), vals.view(np.uint32))
    # larger value -> larger key (pairwise; +0 and the subnormals included)
    for i in range(len(vals)):
        for j in range(len(vals)):
            if vals[i] > vals[j]:
                assert int(keys[i]) > int(keys[j])
    # equal values: the lower index has the larger key
    k_lo = (np.uint64(0x80000000 | 0x3FC00000) << np.uint64(32)) | np.uint64(0xFFFFFFFF - 3)
    k_hi = (np.uint64(0x80000000 | 0x3FC00000) << np.uint64(32)) | np.uint64(0xFFFFFFFF - 9)
    assert k_lo > k_hi and q8.q8_argmax_index(np.array([k_lo]))[0] == 3


def test_packed_bytes(lib):
    f = lib.q8_packed_bytes
    f.restype = ctypes.c_size_t
    f.argtypes = [ctypes.c_int64, ctypes.c_int64]
    # 34 bytes per 32 weights, rows padded to a multiple of 8
    assert f(8, 32) == 8 * 34
    assert f(1152, 896) == 1152 * 896 // 32 * 34
    assert f(1, 64) == 8 * 2 * 34
    assert f(151936, 896) == 151936 * 28 * 34
    assert f(0, 32) == 0 and f(8, 0) == 0 and f(8, 48) == 0 and f(-8, 32) == 0


def test_q6k_packed_bytes(lib):
    f = lib.q8_q6k_packed_bytes
    f.restype = ctypes.c_size_t
    f.argtypes = [ctypes.c_int64, ctypes.c_int64]
    # one 6720-byte unit per (tile of 32 rows, 256-weight block)
    assert f(32, 256) == 6720
    assert f(33, 512) == 2 * 2 * 6720
    assert f(152064, 3584) == 4752 * 14 * 6720
    assert f(0, 256) == 0 and f(8, 300) == 0 and f(8, 0) == 0


def test_status_strings(lib):
    f = lib.q8_status_string
    f.restype = ctypes.c_char_p
    f.argtypes = [ctypes.c_int]
    texts = {f(i).decode() for i in range(8)}
    assert len(texts) == 8 and "ok" in texts
    assert f(99).decode() == "unknown status"


def test_library_targets_sm100a_only():
    from q8_block_quantized_02_b200 import build
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.NVCC_FLAGS)


def test_host_validation_runs_before_any_device_work(lib):
    """Every entry point checks shapes, size limits, null pointers and flags on
    the host before it touches CUDA, so these rejections need no GPU: 2 =
    Q8_ERR_SHAPE, 5 = Q8_ERR_UNSUPPORTED, 1 = Q8_ERR_INVALID."""
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    F = ctypes.c_float

    def fn(name, *argtypes):
        f = getattr(lib, name)
        f.restype = ctypes.c_int
        f.argtypes = list(argtypes)
        return f

    n = None  # null pointer / default stream
    gemv = fn("q8_gemv", P, P, P, I64, I64, I64, P)
    assert gemv(n, n, n, 8, 48, 1, n) == 2          # K % 32
    assert gemv(n, n, n, 0, 32, 1, n) == 2          # M <= 0
    assert gemv(n, n, n, 8, 32, 0, n) == 2          # N <= 0
    assert gemv(n, n, n, 8, 32, 17, n) == 5         # N > 16
    assert gemv(n, n, n, 8, 32, 1, n) == 1          # null W
    res = fn("q8_gemv_residual", P, P, P, P, I64, I64, I64, P)
    assert res(n, n, n, n, 8, 40, 1, n) == 2
    assert res(n, n, n, n, 8, 32, 17, n) == 5
    assert res(n, n, n, n, 8, 32, 2, n) == 1
    am = fn("q8_gemv_argmax", P, P, P, I64, I64, I64, P, P)
    assert am(n, n, n, 8, 33, 1, n, n) == 2
    assert am(n, n, n, 8, 32, 5, n, n) == 5         # N > 4
    assert am(n, n, n, 8, 32, 4, n, n) == 1
    gs = fn("q8_gemv_split", P, P, P, I64, I64, I64, P)
    assert gs(n, n, n, 8, 48, 1, n) == 2
    assert gs(n, n, n, 8, 32, 17, n) == 5
    assert gs(n, n, n, 8, 32, 4, n) == 1
    ss = fn("q8_gate_up_swiglu_split", P, P, P, I64, I64, I64, P)
    assert ss(n, n, n, 12, 32, 1, n) == 2
    assert ss(n, n, n, 16, 32, 17, n) == 5
    assert ss(n, n, n, 16, 32, 8, n) == 1
    sw = fn("q8_gate_up_swiglu", P, P, P, I64, I64, I64, P)
    assert sw(n, n, n, 12, 32, 1, n) == 2           # I % 8
    assert sw(n, n, n, 16, 32, 17, n) == 5
    qa = fn("q8_quantize_act", P, P, P, I64, I64, P)
    assert qa(n, n, n, 1, 31, n) == 2
    rq = fn("q8_rmsnorm_quantize_act", P, P, F, P, P, P, I64, I64, P)
    assert rq(n, n, 1e-6, n, n, n, 1, 48, n) == 2
    assert rq(n, n, -1e-6, n, n, n, 1, 32, n) == 1  # eps < 0
    assert rq(n, n, float("nan"), n, n, n, 1, 32, n) == 1
    assert rq(n, n, float("inf"), n, n, n, 1, 32, n) == 1
    qq = fn("q8q8_gemv", P, P, P, P, I64, I64, I64, P)
    assert qq(n, n, n, n, 8, 16, 1, n) == 2
    assert qq(n, n, n, n, 8, 32, 17, n) == 5
    bd = fn("q8q8_block_dots", P, P, P, I64, I64, I64, P)
    assert bd(n, n, n, 8, 20, 1, n) == 2
    for name in ("q8_q4k_gemv", "q8_q6k_gemv", "q8_q6k_gemv_packed"):
        kq = fn(name, P, P, P, I64, I64, I64, P)
        assert kq(n, n, n, 8, 896, 1, n) == 2       # K % 256
        assert kq(n, n, n, 8, 512, 5, n) == 5       # N > 4
        assert kq(n, n, n, 8, 512, 1, n) == 1
    for name in ("q8_q6k_pack_weights", "q8_q6k_unpack_weights"):
        pk = fn(name, P, I64, I64, P, P)
        assert pk(n, 8, 300, n, n) == 2             # K % 256
        assert pk(n, 0, 256, n, n) == 2             # M <= 0
        assert pk(n, 8, 256, n, n) == 1             # null pointers
    route = fn("q8_moe_route", P, I64, I64, I64, ctypes.c_int, P, P, P)
    assert route(n, 1, 4, 5, 0, n, n, n) == 2       # top_k > E
    assert route(n, 17, 60, 4, 0, n, n, n) == 5     # T > 16
    assert route(n, 1, 60, 4, 2, n, n, n) == 1      # renormalize not 0/1
    moe = fn("q8_moe_gemv", P, P, P, P, P, P, P, P, I64, I64, I64, I64, I64, I64, P, ctypes.c_size_t, P)
    assert moe(n, n, n, n, n, n, n, n, 1, 60, 4, 2000, 1408, 5632, n, 0, n) == 2    # H % 32
    assert moe(n, n, n, n, n, n, n, n, 1, 60, 4, 2048, 1408, 5632, n, 0, n) == 1    # half a shared expert
    noalloc = fn("q8_moe_gemv_noalloc", P, P, P, P, P, P, P, P, I64, I64, I64, I64, I64, I64, P)
    assert noalloc(n, n, n, n, n, n, n, n, 16, 64, 8, 2048, 8192, 32, n) == 5      # scratch too small
    msg = lib.q8_last_cuda_error
    msg.restype = ctypes.c_char_p
    assert b"4194304" in msg()
    # small valid sizes with null buffers: rejected by the argument checks,
    # before the scratch address is looked up or anything is enqueued
    assert noalloc(n, n, n, n, n, n, n, n, 1, 60, 4, 2048, 1408, 5632, n) == 1
    assert noalloc(n, n, n, n, n, n, n, n, 1, 60, 4, 2048, 1408, 0, n) == 1
    assert noalloc(n, n, n, n, n, n, n, n, 1, 60, 4, 2000, 1408, 0, n) == 2          # H % 32
    assert noalloc(n, n, n, n, n, n, n, n, 17, 60, 4, 2048, 1408, 0, n) == 5         # T > 16
    pack = fn("q8_pack_weights", P, I64, I64, P, P)
    assert pack(n, 8, 40, n, n) == 2
    init = fn("q8_moe_workspace_init", P, ctypes.c_size_t, P)
    assert init(n, 0, n) == 2
