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
