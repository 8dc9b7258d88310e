"""ctypes view of ``libtint4.so`` (the C ABI declared in include/tint4.h).

Loading is lazy; a missing or unloadable library raises ``RuntimeError`` at
the first call -- there is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtint4.so")

STATUS = {
    0: "TINT4_OK",
    1: "TINT4_ERR_INVALID_ARG",
    2: "TINT4_ERR_UNSUPPORTED_SHAPE",
    3: "TINT4_ERR_MISALIGNED",
    4: "TINT4_ERR_CUDA",
    5: "TINT4_ERR_TIMEOUT",
    6: "TINT4_ERR_WORKSPACE",
    7: "TINT4_ERR_NO_DEVICE",
}

P = ctypes.c_void_p
I = ctypes.c_int
U64 = ctypes.c_uint64
SZ = ctypes.c_size_t

MAX_GROUPS = 4   # TINT4_MAX_GROUPS


class WeightGroup(ctypes.Structure):
    """tint4_weight_group: one weight matrix of a grouped call (device pointers)."""
    _fields_ = [("w_packed", P), ("row_scale", P), ("bias", P), ("y", P), ("N", I)]

# name -> (restype, argtypes); mirrors include/tint4.h
SIGNATURES = {
    "tint4_abi_version": (I, []),
    "tint4_status_string": (ctypes.c_char_p, [I]),
    "tint4_pack_weights": (I, [P, I, I, I, P, P, P]),
    "convrot_quantize_act": (I, [P, I, I, I, I, P, P, P]),
    "w4a8_gemm": (I, [P, P, P, P, P, P, I, I, I, P]),
    "w4a4_gemm": (I, [P, P, P, P, P, P, I, I, I, P]),
    "w4a4_gemm_widened": (I, [P, P, P, P, P, P, I, I, I, P, SZ, P]),
    "convrot_linear_workspace_size": (SZ, [I, I, I]),
    "convrot_w4a8_linear_workspace": (SZ, [I, I]),
    "convrot_w4a8_linear": (I, [P, P, P, P, P, I, I, I, I, P, SZ, P]),
    "convrot_w4a4_linear": (I, [P, P, P, P, P, I, I, I, I, P, SZ, P]),
    "convrot_w4a8_linear_noalloc": (I, [P, P, P, P, P, I, I, I, I, P]),
    "w4a16_gemv_gemm": (I, [P, P, P, P, I, P, I, I, I, P]),
    "w4a8_gemm_grouped": (I, [P, P, P, I, I, I, P]),
    "tint4_quantize_weights_int8": (I, [P, I, I, I, P, P, P]),
    "w8a8_gemm": (I, [P, P, P, P, P, P, I, I, I, P]),
    "convrot_w8a8_linear": (I, [P, P, P, P, P, I, I, I, I, P, SZ, P]),
    "convrot_w4a8_linear_grouped": (I, [P, P, I, I, I, I, P, SZ, P]),
    "tint4_pack_weights_groupwise": (I, [P, I, I, I, I, P, P, P, P]),
    "w4a8_gemm_groupwise": (I, [P, P, P, P, P, P, P, I, I, I, P]),
    "convrot_w4a8_linear_groupwise": (I, [P, P, P, P, P, P, I, I, I, I, P, SZ, P]),
    "tint4_pack_weights_groupwise_f16": (I, [P, I, I, I, I, P, P, P, P]),
    "w4a8_gemm_groupwise_f16": (I, [P, P, P, P, P, P, P, I, I, I, P]),
    "convrot_w4a8_linear_groupwise_f16": (I, [P, P, P, P, P, P, I, I, I, I, P, SZ, P]),
    "tint4_quantize_weights_int8_f16": (I, [P, I, I, I, P, P, P]),
    "w8a8_gemm_f16": (I, [P, P, P, P, P, P, I, I, I, P]),
    "convrot_w8a8_linear_f16": (I, [P, P, P, P, P, I, I, I, I, P, SZ, P]),
    "tint4_debug_int32_gemm": (I, [P, I, P, P, I, I, I, P]),
    "tint4_debug_w4a8_gemm_even_odd": (I, [P, P, P, P, P, P, I, I, I, P]),
    "tint4_debug_bounded_wait": (I, [U64, P]),
    "tint4_get_device_error": (I, [P]),
    "tint4_set_wait_limit_ns": (I, [U64]),
    "tint4_set_decode_weight_prefetch": (I, [ctypes.c_int]),
}

_lock = threading.Lock()
_lib = None


class Tint4Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        self.name = STATUS.get(status, f"status {status}")
        super().__init__(f"{fn} failed: {self.name}")


def load():
    """The loaded library (raises RuntimeError if it is not built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libtint4.so is not built ({LIB_PATH}); run "
                "`python -m int4_weight_quantized_block_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def call(name: str, *args) -> None:
    rc = getattr(load(), name)(*args)
    if rc != 0:
        raise Tint4Error(name, rc)


def raw(name: str, *args):
    """Call without raising; returns the raw result."""
    return getattr(load(), name)(*args)
