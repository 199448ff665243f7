"""Python binding of libq8 (include/q8.h): Q8_0 decode products on B200.

Argument marshalling only.  Each function forwards to the C entry point of
the same name: torch CUDA tensors are passed by ``data_ptr()`` (plain integer
device addresses are accepted too), ``stream`` defaults to torch's current
stream, and a non-zero status raises :class:`Q8Error`.  Every step of the
computation runs in the CUDA library; there is no fallback path.  If
``libq8.so`` is missing or cannot be loaded, every call raises.

Build the library with ``python -m q8_block_quantized_02_b200.build`` (or
``__graft_entry__.build()``).
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = [
    "Q8Error", "lib_path", "q8_status_string", "q8_last_cuda_error", "q8_read_device_error",
    "q8_version", "q8_packed_bytes", "q8_pack_weights", "q8_unpack_weights", "q8_gemv",
    "q8_gemv_residual", "q8_gemv_argmax", "q8_argmax_index", "q8_argmax_value",
    "q8_q4k_gemv", "q8_q6k_gemv",
    "q8_q6k_packed_bytes", "q8_q6k_pack_weights", "q8_q6k_unpack_weights", "q8_q6k_gemv_packed",
    "q8_gate_up_swiglu", "q8_moe_route", "q8_moe_workspace_bytes", "q8_moe_workspace_init",
    "q8_moe_gemv",
    "q8_moe_gemv_noalloc",
    "q8_quantize_act", "q8_rmsnorm_quantize_act", "q8q8_gemv", "q8q8_block_dots",
    "q8_test_wait_timeout", "q8_gemv_split", "q8_gate_up_swiglu_split",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_lock = threading.Lock()
_lib = None

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_INT = ctypes.c_int
_SZ = ctypes.c_size_t

# name -> (restype, argtypes); mirrors include/q8.h
_SIGS = {
    "q8_status_string": (ctypes.c_char_p, [_INT]),
    "q8_last_cuda_error": (ctypes.c_char_p, []),
    "q8_read_device_error": (_INT, [ctypes.POINTER(ctypes.c_uint32)]),
    "q8_version": (_INT, []),
    "q8_packed_bytes": (_SZ, [_I64, _I64]),
    "q8_pack_weights": (_INT, [_P, _I64, _I64, _P, _P]),
    "q8_unpack_weights": (_INT, [_P, _I64, _I64, _P, _P]),
    "q8_gemv": (_INT, [_P, _P, _P, _I64, _I64, _I64, _P]),
    "q8_gemv_argmax": (_INT, [_P, _P, _P, _I64, _I64, _I64, _P, _P]),
    "q8_gemv_residual": (_INT, [_P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "q8_q4k_gemv": (_INT, [_P, _P, _P, _I64, _I64, _I64, _P]),
    "q8_q6k_gemv": (_INT, [_P, _P, _P, _I64, _I64, _I64, _P]),
    "q8_q6k_packed_bytes": (_SZ, [_I64, _I64]),
    "q8_q6k_pack_weights": (_INT, [_P, _I64, _I64, _P, _P]),
    "q8_q6k_unpack_weights": (_INT, [_P, _I64, _I64, _P, _P]),
    "q8_q6k_gemv_packed": (_INT, [_P, _P, _P, _I64, _I64, _I64, _P]),
    "q8_gate_up_swiglu": (_INT, [_P, _P, _P, _I64, _I64, _I64, _P]),
    "q8_moe_route": (_INT, [_P, _I64, _I64, _I64, _INT, _P, _P, _P]),
    "q8_moe_workspace_bytes": (_SZ, [_I64, _I64, _I64, _I64, _I64, _I64]),
    "q8_moe_workspace_init": (_INT, [_P, _SZ, _P]),
    "q8_moe_gemv": (_INT, [_P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, _I64,
                           _P, _SZ, _P]),
    "q8_moe_gemv_noalloc": (_INT, [_P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64,
                                   _I64, _P]),
    "q8_quantize_act": (_INT, [_P, _P, _P, _I64, _I64, _P]),
    "q8q8_gemv": (_INT, [_P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "q8_rmsnorm_quantize_act": (_INT, [_P, _P, ctypes.c_float, _P, _P, _P, _I64, _I64, _P]),
    "q8q8_block_dots": (_INT, [_P, _P, _P, _I64, _I64, _I64, _P]),
    "q8_test_wait_timeout": (_INT, [ctypes.c_uint32, _P, _P]),
    "q8_gemv_split": (_INT, [_P, _P, _P, _I64, _I64, _I64, _P]),
    "q8_gate_up_swiglu_split": (_INT, [_P, _P, _P, _I64, _I64, _I64, _P]),
}


class Q8Error(RuntimeError):
    """A libq8 call returned a non-zero q8_status."""

    def __init__(self, func: str, status: int):
        lib = _load()
        text = lib.q8_status_string(status).decode()
        detail = lib.q8_last_cuda_error().decode() if status == 6 else ""
        super().__init__(f"{func}: {text}" + (f" [{detail}]" if detail else ""))
        self.status = status


def lib_path() -> str:
    return os.path.join(_HERE, "libq8.so")


def _load():
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            path = lib_path()
            if not os.path.exists(path):
                raise RuntimeError(f"libq8.so is not built ({path}); run "
                                   "`python -m q8_block_quantized_02_b200.build`")
            lib = ctypes.CDLL(path)
            for name, (res, args) in _SIGS.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _call(name, *args):
    st = getattr(_load(), name)(*args)
    if st != 0:
        raise Q8Error(name, st)


def q8_status_string(status: int) -> str:
    return _load().q8_status_string(int(status)).decode()


def q8_last_cuda_error() -> str:
    return _load().q8_last_cuda_error().decode()


def q8_read_device_error():
    """Synchronise the device; return (status, raw word) and clear the word."""
    w = ctypes.c_uint32(0)
    st = _load().q8_read_device_error(ctypes.byref(w))
    return st, w.value


def q8_version() -> int:
    return _load().q8_version()


def q8_packed_bytes(M: int, K: int) -> int:
    return int(_load().q8_packed_bytes(M, K))


def q8_pack_weights(gguf_blocks, M, K, packed, stream=None):
    _call("q8_pack_weights", _ptr(gguf_blocks), M, K, _ptr(packed), _stream(stream))


def q8_unpack_weights(packed, M, K, gguf_blocks, stream=None):
    _call("q8_unpack_weights", _ptr(packed), M, K, _ptr(gguf_blocks), _stream(stream))


def q8_gemv(W, x, y, M, K, N, stream=None):
    _call("q8_gemv", _ptr(W), _ptr(x), _ptr(y), M, K, N, _stream(stream))


def q8_q4k_gemv(W, x, y, M, K, N, stream=None):
    """W: raw GGUF Q4_K blocks (uint8 device tensor)."""
    _call("q8_q4k_gemv", _ptr(W), _ptr(x), _ptr(y), M, K, N, _stream(stream))


def q8_q6k_gemv(W, x, y, M, K, N, stream=None):
    """W: raw GGUF Q6_K blocks (uint8 device tensor)."""
    _call("q8_q6k_gemv", _ptr(W), _ptr(x), _ptr(y), M, K, N, _stream(stream))


def q8_q6k_packed_bytes(M: int, K: int) -> int:
    return int(_load().q8_q6k_packed_bytes(M, K))


def q8_q6k_pack_weights(raw, M, K, packed, stream=None):
    """raw GGUF Q6_K blocks -> the tile kernel's 6720-byte units."""
    _call("q8_q6k_pack_weights", _ptr(raw), M, K, _ptr(packed), _stream(stream))


def q8_q6k_unpack_weights(packed, M, K, raw, stream=None):
    _call("q8_q6k_unpack_weights", _ptr(packed), M, K, _ptr(raw), _stream(stream))


def q8_q6k_gemv_packed(packed, x, y, M, K, N, stream=None):
    """packed: q8_q6k_pack_weights output (uint8 device tensor)."""
    _call("q8_q6k_gemv_packed", _ptr(packed), _ptr(x), _ptr(y), M, K, N, _stream(stream))


def q8_gemv_residual(W, x, residual, y, M, K, N, stream=None):
    """y = W x + residual; residual may be y itself."""
    _call("q8_gemv_residual", _ptr(W), _ptr(x), _ptr(residual), _ptr(y), M, K, N, _stream(stream))


def q8_gemv_argmax(W, x, y, M, K, N, best, stream=None):
    """y may be None (logits not written); best: [N] uint64 keys (torch.int64
    or uint64 tensor), decoded by q8_argmax_index / q8_argmax_value."""
    _call("q8_gemv_argmax", _ptr(W), _ptr(x), None if y is None else _ptr(y), M, K, N, _ptr(best),
          _stream(stream))


def q8_argmax_index(keys):
    """Row index held in q8_gemv_argmax keys (numpy array or scalar; the
    header's q8_argmax_index)."""
    import numpy as np
    k = np.asarray(keys).astype(np.uint64)
    return (np.uint64(0xFFFFFFFF) - (k & np.uint64(0xFFFFFFFF))).astype(np.int64)


def q8_argmax_value(keys):
    """Maximum value held in q8_gemv_argmax keys, as float32 (the header's
    q8_argmax_value)."""
    import numpy as np
    h = (np.asarray(keys).astype(np.uint64) >> np.uint64(32)).astype(np.uint32)
    u = np.where(h & np.uint32(0x80000000), h & np.uint32(0x7FFFFFFF), ~h).astype(np.uint32)
    return u.view(np.float32)


def q8_gate_up_swiglu(W, x, h, I, K, N, stream=None):
    _call("q8_gate_up_swiglu", _ptr(W), _ptr(x), _ptr(h), I, K, N, _stream(stream))


def q8_moe_route(logits, T, E, top_k, renormalize, idx, w, stream=None):
    _call("q8_moe_route", _ptr(logits), T, E, top_k, int(renormalize), _ptr(idx), _ptr(w),
          _stream(stream))


def q8_moe_workspace_bytes(T, E, top_k, H, I, I_shared) -> int:
    return int(_load().q8_moe_workspace_bytes(T, E, top_k, H, I, I_shared))


def q8_moe_workspace_init(workspace, workspace_bytes, stream=None):
    _call("q8_moe_workspace_init", _ptr(workspace), int(workspace_bytes), _stream(stream))


def q8_moe_gemv(gate_up_experts, down_experts, shared_gate_up, shared_down, idx, w, x, y, T, E,
                top_k, H, I, I_shared, workspace, workspace_bytes, stream=None):
    _call("q8_moe_gemv", _ptr(gate_up_experts), _ptr(down_experts), _ptr(shared_gate_up),
          _ptr(shared_down), _ptr(idx), _ptr(w), _ptr(x), _ptr(y), T, E, top_k, H, I, I_shared,
          _ptr(workspace), int(workspace_bytes), _stream(stream))


def q8_moe_gemv_noalloc(gate_up_experts, down_experts, shared_gate_up, shared_down, idx, w, x, y,
                        T, E, top_k, H, I, I_shared, stream=None):
    _call("q8_moe_gemv_noalloc", _ptr(gate_up_experts), _ptr(down_experts), _ptr(shared_gate_up),
          _ptr(shared_down), _ptr(idx), _ptr(w), _ptr(x), _ptr(y), T, E, top_k, H, I, I_shared,
          _stream(stream))


def q8_quantize_act(x, xq, xd, N, K, stream=None):
    _call("q8_quantize_act", _ptr(x), _ptr(xq), _ptr(xd), N, K, _stream(stream))


def q8_rmsnorm_quantize_act(x, gamma, eps, xq, xd, rinv, N, K, stream=None):
    """rinv may be None."""
    _call("q8_rmsnorm_quantize_act", _ptr(x), _ptr(gamma), float(eps), _ptr(xq), _ptr(xd), _ptr(rinv),
          N, K, _stream(stream))


def q8q8_gemv(W, xq, xd, y, M, K, N, stream=None):
    _call("q8q8_gemv", _ptr(W), _ptr(xq), _ptr(xd), _ptr(y), M, K, N, _stream(stream))


def q8q8_block_dots(W, xq, dots, M, K, N, stream=None):
    _call("q8q8_block_dots", _ptr(W), _ptr(xq), _ptr(dots), M, K, N, _stream(stream))


def q8_test_wait_timeout(limit_us, out, stream=None):
    _call("q8_test_wait_timeout", int(limit_us), _ptr(out), _stream(stream))


def q8_gemv_split(W, x, y, M, K, N, stream=None):
    _call("q8_gemv_split", _ptr(W), _ptr(x), _ptr(y), M, K, N, _stream(stream))


def q8_gate_up_swiglu_split(W, x, h, I, K, N, stream=None):
    _call("q8_gate_up_swiglu_split", _ptr(W), _ptr(x), _ptr(h), I, K, N, _stream(stream))
