"""CPU oracle for the packed-INT4 ConvRot quantized linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The product library never imports, links or calls it, and it never
imports the product: the two share no code.

The arithmetic lives in ``tint4_oracle.c`` (plain C, OpenMP over rows); this
module only compiles it on first use and marshals numpy arrays through ctypes.
Every function states which page passage it restates; the C file's header
lists the readings taken where the pages are silent.

Parity status: every function here is pinned by a ``-m "not gpu"`` test to
something other than itself (closed forms, invariants, brute force, worked
examples derived by hand in ``tests/golden/``).  None is pinned to a number
printed by the pages, because the pages print no tensors.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tint4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liboracle.so`` (gcc, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", "-Wall", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        I = ctypes.c_int
        L = ctypes.c_long
        sig = {
            "oracle_hadamard": [I, P],
            "oracle_fwht_f32": [P, I],
            "oracle_rotate_rows_f32": [P, L, I, I],
            "oracle_pack_int4": [P, L, I, P],
            "oracle_unpack_int4": [P, L, I, P],
            "oracle_pack_weights": [P, I, I, I, P, P, P],
            "oracle_quantize_act": [P, I, I, I, I, P, P, P],
            "oracle_gemm_i32": [P, P, I, I, I, P],
            "oracle_gemm_i32_sampled": [P, P, I, P, L, P],
            "oracle_epilogue": [P, P, P, P, I, I, P],
            "oracle_epilogue_f64": [P, P, P, P, I, I, P],
            "oracle_epilogue_sampled": [P, P, P, P, P, L, P],
            "oracle_epilogue_sampled_f64": [P, P, P, P, P, L, P],
            "oracle_convrot_linear": [P, P, P, P, I, I, I, I, I, P],
            "oracle_convrot_linear_f64": [P, P, P, P, I, I, I, I, I, P],
            "oracle_w4a16": [P, P, P, P, I, I, I, I, P],
            "oracle_w4a16_f64": [P, P, P, P, I, I, I, I, P],
            "oracle_w4a16_dequant_f64": [P, P, P, P, I, I, I, I, P],
            "oracle_w4a16_weights_f64": [P, P, P, I, I, I, I, P],
            "oracle_quantize_weights_int8": [P, I, I, I, P, P],
            "oracle_quantize_weights_int8_ex": [P, I, I, I, I, P, P],
            "oracle_pack_weights_groupwise": [P, I, I, I, I, I, P, P, P, P],
            "oracle_pack_weights_groupwise_ex": [P, I, I, I, I, I, I, P, P, P, P],
            "oracle_round_f16": [P, L, P],
            "oracle_gemm_groupwise_f64": [P, P, P, P, P, P, I, I, I, I, P, P],
            "oracle_gemm_groupwise_sampled_f64": [P, P, P, P, P, P, I, I, I, I, P, L, P, P],
            "oracle_round_bf16": [P, L, P],
            "oracle_num_threads": [],
        }
        for name, args in sig.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = I
        lib.oracle_double_to_bf16.argtypes = [ctypes.c_double]
        lib.oracle_double_to_bf16.restype = ctypes.c_uint16
        _lib = lib
        return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"{name}: oracle rejected its arguments (rc={rc})")


def num_threads() -> int:
    """OpenMP threads the oracle uses."""
    return int(_load().oracle_num_threads())


# --------------------------------------------------------------------------
# bf16 helpers (the oracle's own; inputs arrive as raw bf16 bits, uint16)
# --------------------------------------------------------------------------

def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float32 values, exactly."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def double_to_bf16_bits(v: float) -> int:
    """Round one double to the nearest bf16 (ties to even), return its bits."""
    return int(_load().oracle_double_to_bf16(float(v)))


def round_bf16(v: np.ndarray) -> np.ndarray:
    """Round an fp64 array to bf16 bits (nearest, ties to even), same shape."""
    a = _c(v, np.float64)
    out = np.empty(a.shape, dtype=np.uint16)
    _check(_load().oracle_round_bf16(_ptr(a), a.size, _ptr(out)), "round_bf16")
    return out


# --------------------------------------------------------------------------
# Rotation
# --------------------------------------------------------------------------

def hadamard(g: int) -> np.ndarray:
    """Orthonormal Sylvester Hadamard matrix H_g (fp64, g x g), natural order.

    The matrix behind the rotation the pages call Hadamard / QuaRot / ConvRot
    ("ComfyUI-INT-Crush", "Inference > INT4 > CUDA backend"; "TINT4 v1.2",
    "参数选择指南" enable_quarot)."""
    H = np.empty((g, g), dtype=np.float64)
    _check(_load().oracle_hadamard(g, _ptr(H)), "hadamard")
    return H


def fwht_f32(v: np.ndarray) -> np.ndarray:
    """Orthonormal fast Walsh-Hadamard transform of one fp32 block (copy)."""
    out = _c(v, np.float32).copy()
    _check(_load().oracle_fwht_f32(_ptr(out), out.size), "fwht_f32")
    return out


def rotate_rows_f32(rows: np.ndarray, g: int) -> np.ndarray:
    """Rotate every length-g block along the last axis (fp32, copy).

    "ComfyUI-INT-Crush", "Forward Pass" step 2 (rotate activations with the
    layer's rot_size); the same block rotation is applied to W offline."""
    out = _c(rows, np.float32).copy()
    K = out.shape[-1]
    n = out.size // K
    _check(_load().oracle_rotate_rows_f32(_ptr(out), n, K, g), "rotate_rows_f32")
    return out


# --------------------------------------------------------------------------
# Packing
# --------------------------------------------------------------------------

def pack_int4(codes: np.ndarray) -> np.ndarray:
    """int8 codes [R, K] -> uint8 [R, K/2], code 2j in the low nibble of byte j.

    "ComfyUI-INT-Crush", "Weight Format" (uint8, 2 per byte)."""
    q = _c(codes, np.int8)
    R, K = q.shape
    out = np.empty((R, K // 2), dtype=np.uint8)
    _check(_load().oracle_pack_int4(_ptr(q), R, K, _ptr(out)), "pack_int4")
    return out


def unpack_int4(packed: np.ndarray) -> np.ndarray:
    """uint8 [R, K/2] -> int8 codes [R, K] (two's complement nibbles)."""
    p = _c(packed, np.uint8)
    R, Kh = p.shape
    out = np.empty((R, 2 * Kh), dtype=np.int8)
    _check(_load().oracle_unpack_int4(_ptr(p), R, 2 * Kh, _ptr(out)), "unpack_int4")
    return out


# --------------------------------------------------------------------------
# Quantization
# --------------------------------------------------------------------------

def pack_weights(W: np.ndarray, g: int):
    """Twin of ``tint4_pack_weights``: rotate W along K, per-row symmetric int4.

    Returns (packed uint8 [N, K/2], row_scale fp32 [N], codes int8 [N, K]).
    "ComfyUI-INT-Crush", "Weight Format"; "feat: packed int4 convrot model
    loading and dispatch", "Summary" (packed nibbles + row scales)."""
    Wc = _c(W, np.float32)
    N, K = Wc.shape
    packed = np.empty((N, K // 2), dtype=np.uint8)
    scale = np.empty(N, dtype=np.float32)
    codes = np.empty((N, K), dtype=np.int8)
    _check(_load().oracle_pack_weights(_ptr(Wc), N, K, g, _ptr(packed), _ptr(scale),
                                       _ptr(codes)), "pack_weights")
    return packed, scale, codes


def quantize_weights_int8(W: np.ndarray, g: int, scale_f16: bool = False):
    """Twin of ``tint4_quantize_weights_int8``: rotate W along K, per-row
    symmetric int8 codes [N, K] in [-127, 127] and fp32 row scales [N].

    "ComfyUI-INT-Crush", "Inference > INT8" (int8 weights x int8 activations,
    int32 accumulation); the rotation and rounding are those of the int4
    weights ("Weight Format", "Forward Pass").  scale_f16 (twin of
    ``tint4_quantize_weights_int8_f16``; "Weight Format": INT8 scales fp16
    [out, 1]): each scale is rounded to fp16 and the codes are taken against
    that stored scale; the scales come back as float32 values on the fp16
    grid (``f16_bits`` gives their bit patterns)."""
    Wc = _c(W, np.float32)
    N, K = Wc.shape
    codes = np.empty((N, K), dtype=np.int8)
    scale = np.empty(N, dtype=np.float32)
    _check(_load().oracle_quantize_weights_int8_ex(_ptr(Wc), N, K, g, int(scale_f16), _ptr(codes),
                                                   _ptr(scale)), "quantize_weights_int8")
    return codes, scale


def round_f16(v: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest fp16 number (ties to even; from
    65520 on infinity), returned as float32."""
    a = _c(v, np.float32)
    out = np.empty(a.shape, dtype=np.float32)
    _check(_load().oracle_round_f16(_ptr(a), a.size, _ptr(out)), "round_f16")
    return out


def f16_bits(v: np.ndarray) -> np.ndarray:
    """IEEE fp16 bit patterns (uint16) of float32 values that lie on the fp16
    grid (the oracle's fp16 scales): sign bit, 5-bit biased exponent, 10-bit
    fraction; subnormals are multiples of 2^-24."""
    a = np.asarray(v, np.float32)
    mag = np.abs(a.astype(np.float64))
    finite = np.isfinite(mag)
    m = np.where(finite, mag, 1.0)
    e = np.floor(np.log2(np.where(m > 0, m, 1.0)))
    normal = finite & (m >= 2.0 ** -14)
    frac_n = np.where(normal, m / 2.0 ** e - 1.0, 0.0) * 1024.0
    sub_n = np.where(finite & ~normal, m * 2.0 ** 24, 0.0)
    if np.any(np.isnan(a)) or np.any(finite & (mag > 65504.0)) or \
            np.any(frac_n != np.rint(frac_n)) or np.any(sub_n != np.rint(sub_n)):
        raise ValueError("values not on the fp16 grid")
    out = np.where(normal, ((e.astype(np.int64) + 15) << 10) | frac_n.astype(np.int64),
                   sub_n.astype(np.int64))
    out = np.where(finite, out, 0x7C00)
    return (out | np.where(np.signbit(a), 0x8000, 0)).astype(np.uint16)


def quantize_act(x_bits: np.ndarray, g: int, bits: int):
    """Twin of ``convrot_quantize_act``: rotate x then per-token symmetric codes.

    x_bits: bf16 bit patterns uint16 [M, K].  Returns (codes int8 [M, K],
    tok_scale fp32 [M], packed uint8 [M, K/2] or None for bits == 8).
    "ComfyUI-INT-Crush", "Inference > INT4 > Triton backend" (dynamic
    activation quantization) and "Forward Pass" steps 2 and 5."""
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    codes = np.empty((M, K), dtype=np.int8)
    scale = np.empty(M, dtype=np.float32)
    packed = np.empty((M, K // 2), dtype=np.uint8) if bits == 4 else None
    _check(_load().oracle_quantize_act(_ptr(x), M, K, g, bits, _ptr(codes), _ptr(scale),
                                       _ptr(packed)), "quantize_act")
    return codes, scale, packed


# --------------------------------------------------------------------------
# GEMM, epilogue, whole layer
# --------------------------------------------------------------------------

def gemm_i32(a: np.ndarray, w: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k a[m, k] w[n, k] (exact int32).

    "ComfyUI-INT-Crush", "Inference > INT4 > CUDA backend" (INT8 GEMM)."""
    ac, wc = _c(a, np.int8), _c(w, np.int8)
    M, K = ac.shape
    N = wc.shape[0]
    out = np.empty((M, N), dtype=np.int32)
    _check(_load().oracle_gemm_i32(_ptr(ac), _ptr(wc), M, N, K, _ptr(out)), "gemm_i32")
    return out


def gemm_i32_sampled(a: np.ndarray, w: np.ndarray, pairs: np.ndarray) -> np.ndarray:
    """The same sums for selected (m, n) pairs only (pairs int64 [P, 2])."""
    ac, wc = _c(a, np.int8), _c(w, np.int8)
    pr = _c(pairs, np.int64)
    out = np.empty(pr.shape[0], dtype=np.int32)
    _check(_load().oracle_gemm_i32_sampled(_ptr(ac), _ptr(wc), ac.shape[1], _ptr(pr),
                                           pr.shape[0], _ptr(out)), "gemm_i32_sampled")
    return out


def epilogue(acc, tok_scale, row_scale, bias_bits=None) -> np.ndarray:
    """y = bf16(acc * s_tok * s_row (+ bias)) in fp64; returns bf16 bits.

    "ComfyUI-INT-Crush", "Inference > INT4 > CUDA backend" (fused dequant)."""
    A = _c(acc, np.int32)
    M, N = A.shape
    st, sr = _c(tok_scale, np.float32), _c(row_scale, np.float32)
    b = None if bias_bits is None else _c(bias_bits, np.uint16)
    y = np.empty((M, N), dtype=np.uint16)
    _check(_load().oracle_epilogue(_ptr(A), _ptr(st), _ptr(sr), _ptr(b), M, N, _ptr(y)),
           "epilogue")
    return y


def epilogue_f64(acc, tok_scale, row_scale, bias_bits=None) -> np.ndarray:
    """The epilogue's value before the bf16 rounding (fp64)."""
    A = _c(acc, np.int32)
    M, N = A.shape
    st, sr = _c(tok_scale, np.float32), _c(row_scale, np.float32)
    b = None if bias_bits is None else _c(bias_bits, np.uint16)
    y = np.empty((M, N), dtype=np.float64)
    _check(_load().oracle_epilogue_f64(_ptr(A), _ptr(st), _ptr(sr), _ptr(b), M, N, _ptr(y)),
           "epilogue_f64")
    return y


def epilogue_sampled_f64(acc, tok_scale, row_scale, pairs, bias_bits=None) -> np.ndarray:
    """Unrounded epilogue for selected (m, n) pairs (fp64)."""
    A = _c(acc, np.int32)
    st, sr = _c(tok_scale, np.float32), _c(row_scale, np.float32)
    pr = _c(pairs, np.int64)
    b = None if bias_bits is None else _c(bias_bits, np.uint16)
    y = np.empty(pr.shape[0], dtype=np.float64)
    _check(_load().oracle_epilogue_sampled_f64(_ptr(A), _ptr(st), _ptr(sr), _ptr(b), _ptr(pr),
                                               pr.shape[0], _ptr(y)), "epilogue_sampled_f64")
    return y


def epilogue_sampled(acc, tok_scale, row_scale, pairs, bias_bits=None) -> np.ndarray:
    """Epilogue for selected (m, n) pairs; acc holds their sums in pair order."""
    A = _c(acc, np.int32)
    st, sr = _c(tok_scale, np.float32), _c(row_scale, np.float32)
    pr = _c(pairs, np.int64)
    b = None if bias_bits is None else _c(bias_bits, np.uint16)
    y = np.empty(pr.shape[0], dtype=np.uint16)
    _check(_load().oracle_epilogue_sampled(_ptr(A), _ptr(st), _ptr(sr), _ptr(b), _ptr(pr),
                                           pr.shape[0], _ptr(y)), "epilogue_sampled")
    return y


def convrot_linear(x_bits, w_packed, row_scale, g, act_bits, bias_bits=None) -> np.ndarray:
    """Twin of ``convrot_w4a8_linear`` (act_bits 8) / ``convrot_w4a4_linear`` (4).

    Rotate + quantize x, unpack W, int32 GEMM, fused dequant; bf16 bits out.
    "ComfyUI-INT-Crush", "Inference > INT4 > CUDA backend" (fused ConvRot path)."""
    x = _c(x_bits, np.uint16)
    wp = _c(w_packed, np.uint8)
    sr = _c(row_scale, np.float32)
    b = None if bias_bits is None else _c(bias_bits, np.uint16)
    M, K = x.shape
    N = wp.shape[0]
    y = np.empty((M, N), dtype=np.uint16)
    _check(_load().oracle_convrot_linear(_ptr(x), _ptr(wp), _ptr(sr), _ptr(b), M, N, K, g,
                                         act_bits, _ptr(y)), "convrot_linear")
    return y


def convrot_linear_f64(x_bits, w_packed, row_scale, g, act_bits, bias_bits=None) -> np.ndarray:
    """The fused linear's value before the bf16 rounding (fp64)."""
    x = _c(x_bits, np.uint16)
    wp = _c(w_packed, np.uint8)
    sr = _c(row_scale, np.float32)
    b = None if bias_bits is None else _c(bias_bits, np.uint16)
    M, K = x.shape
    N = wp.shape[0]
    y = np.empty((M, N), dtype=np.float64)
    _check(_load().oracle_convrot_linear_f64(_ptr(x), _ptr(wp), _ptr(sr), _ptr(b), M, N, K, g,
                                             act_bits, _ptr(y)), "convrot_linear_f64")
    return y


# --------------------------------------------------------------------------
# Group-wise W4A8 (per row and K group weight scales; symmetric or asymmetric)
# --------------------------------------------------------------------------

def pack_weights_groupwise(W: np.ndarray, g: int, G: int = 128, asym: bool = False,
                           scale_f16: bool = False):
    """Twin of ``tint4_pack_weights_groupwise``: rotate W along K, then int4
    codes per (row, G-wide K group).

    Returns (packed uint8 [N, K/2], scale fp32 [N, K/G], zero uint8 [N, K/G]
    or None, codes int8 [N, K]).  "ComfyUI-INT-Crush", "Weight Format"
    (scales [out, num_groups]); "feat: packed int4 convrot model loading and
    dispatch", "Summary" (the asymmetric W4A8 format).  scale_f16 (twin of
    ``tint4_pack_weights_groupwise_f16``; "Weight Format": the scales are
    stored as fp16): each group scale is rounded to fp16 first and the zero
    point and codes are taken against that stored scale; the scales come back
    as float32 values on the fp16 grid."""
    Wc = _c(W, np.float32)
    N, K = Wc.shape
    packed = np.empty((N, K // 2), dtype=np.uint8)
    scale = np.empty((N, K // G), dtype=np.float32)
    zero = np.empty((N, K // G), dtype=np.uint8) if asym else None
    codes = np.empty((N, K), dtype=np.int8)
    _check(_load().oracle_pack_weights_groupwise_ex(_ptr(Wc), N, K, g, G, int(asym),
                                                    int(scale_f16), _ptr(packed), _ptr(scale),
                                                    _ptr(zero), _ptr(codes)),
           "pack_weights_groupwise")
    return packed, scale, zero, codes


def gemm_groupwise_f64(a, tok_scale, w_packed, scale, zero=None, bias_bits=None, G: int = 128):
    """y = s_tok * sum_j s[n, j] * sum_{k in j} a (q - z) (+ bias), unrounded
    (fp64), and the magnitude of its terms (fp64), both [M, N]."""
    ac = _c(a, np.int8)
    st, sc = _c(tok_scale, np.float32), _c(scale, np.float32)
    wp = _c(w_packed, np.uint8)
    z = None if zero is None else _c(zero, np.uint8)
    b = None if bias_bits is None else _c(bias_bits, np.uint16)
    M, K = ac.shape
    N = wp.shape[0]
    y = np.empty((M, N), dtype=np.float64)
    mag = np.empty((M, N), dtype=np.float64)
    _check(_load().oracle_gemm_groupwise_f64(_ptr(ac), _ptr(st), _ptr(wp), _ptr(sc), _ptr(z),
                                             _ptr(b), M, N, K, G, _ptr(y), _ptr(mag)),
           "gemm_groupwise_f64")
    return y, mag


def gemm_groupwise_sampled_f64(a, tok_scale, w_packed, scale, pairs, zero=None, bias_bits=None,
                               G: int = 128):
    """The same for selected (m, n) pairs (pairs int64 [P, 2]): (y, mag) [P]."""
    ac = _c(a, np.int8)
    st, sc = _c(tok_scale, np.float32), _c(scale, np.float32)
    wp = _c(w_packed, np.uint8)
    z = None if zero is None else _c(zero, np.uint8)
    b = None if bias_bits is None else _c(bias_bits, np.uint16)
    pr = _c(pairs, np.int64)
    M, K = ac.shape
    N = wp.shape[0]
    y = np.empty(pr.shape[0], dtype=np.float64)
    mag = np.empty(pr.shape[0], dtype=np.float64)
    _check(_load().oracle_gemm_groupwise_sampled_f64(_ptr(ac), _ptr(st), _ptr(wp), _ptr(sc),
                                                     _ptr(z), _ptr(b), M, N, K, G, _ptr(pr),
                                                     pr.shape[0], _ptr(y), _ptr(mag)),
           "gemm_groupwise_sampled_f64")
    return y, mag


def w4a16_f64(x_bits, q_packed, scale_bits, zero, group) -> np.ndarray:
    """The W4A16 layer's value before the bf16 rounding (fp64 accumulation)."""
    x = _c(x_bits, np.uint16)
    q = _c(q_packed, np.uint8)
    s = _c(scale_bits, np.uint16)
    z = _c(zero, np.uint8)
    M, K = x.shape
    N = q.shape[0]
    y = np.empty((M, N), dtype=np.float64)
    _check(_load().oracle_w4a16_f64(_ptr(x), _ptr(q), _ptr(s), _ptr(z), M, N, K, group,
                                    _ptr(y)), "w4a16_f64")
    return y


def w4a16_dequant_f64(x_bits, q_packed, scale_bits, zero, group) -> np.ndarray:
    """The W4A16 layer in its 16-bit unpack + 16-bit GEMM form, before the
    output's bf16 rounding: each weight is first rounded to the bf16 number
    nearest to (q - z) * s, then y = x . w^T in fp64.

    "ComfyUI-INT-Crush", "Inference > INT4 > Triton backend": with
    rot_size == 0 the INT4 weights are widened to 16 bits for a 16-bit GEMM;
    "TINT4 v1.2", "v1.1 新特性 > 5": the torchao layer's _qdata/_scale/_zp."""
    x = _c(x_bits, np.uint16)
    q = _c(q_packed, np.uint8)
    s = _c(scale_bits, np.uint16)
    z = _c(zero, np.uint8)
    M, K = x.shape
    N = q.shape[0]
    y = np.empty((M, N), dtype=np.float64)
    _check(_load().oracle_w4a16_dequant_f64(_ptr(x), _ptr(q), _ptr(s), _ptr(z), M, N, K, group,
                                            _ptr(y)), "w4a16_dequant_f64")
    return y


def w4a16_weights_f64(q_packed, scale_bits, zero, group, widen: bool = False) -> np.ndarray:
    """The W4A16 weights, fp64 [N, K]: (q - z) * s exactly, or (widen) that
    product rounded once to bf16 (the 16-bit unpack form of
    ``w4a16_dequant_f64``).  For shapes where the per-output loops are slow,
    ``bf16_bits_to_f32(x) @ w.T`` (a library matrix product) gives the same
    layer values up to fp64 rounding."""
    q = _c(q_packed, np.uint8)
    s = _c(scale_bits, np.uint16)
    z = _c(zero, np.uint8)
    N, K = q.shape[0], 2 * q.shape[1]
    w = np.empty((N, K), dtype=np.float64)
    _check(_load().oracle_w4a16_weights_f64(_ptr(q), _ptr(s), _ptr(z), N, K, group, int(widen),
                                            _ptr(w)), "w4a16_weights_f64")
    return w


def w4a16(x_bits, q_packed, scale_bits, zero, group) -> np.ndarray:
    """Twin of ``w4a16_gemv_gemm``: y = x . ((q - z) * s)^T, fp64 accumulation.

    "TINT4 v1.2", "v1.1 新特性 > 5" (_qdata/_scale/_zp) and "参数选择指南"
    (group_size 128 standard); "ComfyUI-INT-Crush", "Inference > INT4 >
    Triton backend" (W4A16 when rot_size == 0)."""
    x = _c(x_bits, np.uint16)
    q = _c(q_packed, np.uint8)
    s = _c(scale_bits, np.uint16)
    z = _c(zero, np.uint8)
    M, K = x.shape
    N = q.shape[0]
    y = np.empty((M, N), dtype=np.uint16)
    _check(_load().oracle_w4a16(_ptr(x), _ptr(q), _ptr(s), _ptr(z), M, N, K, group, _ptr(y)),
           "w4a16")
    return y
