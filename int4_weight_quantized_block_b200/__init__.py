"""Packed-INT4 ConvRot quantized linear layer for B200 (sm_100a).

Thin Python binding of the C ABI in ``include/tint4.h``: every function here
has the name of the C entry point it calls, checks dtypes / devices /
contiguity, allocates outputs with torch when the caller passes none, and
hands raw pointers plus the current CUDA stream to ``libtint4.so``.  All of
the arithmetic runs in the library's CUDA kernels; there is no Python or CPU
fallback (a missing library raises).
"""
from __future__ import annotations

from typing import Optional, Tuple

import ctypes

import torch

from . import _native
from ._native import Tint4Error

__all__ = [
    "Tint4Error",
    "tint4_pack_weights",
    "convrot_quantize_act",
    "w4a8_gemm",
    "w4a4_gemm",
    "convrot_linear_workspace_size",
    "w4a4_gemm_widened",
    "convrot_w4a8_linear",
    "convrot_w4a4_linear",
    "convrot_w4a8_linear_noalloc",
    "w4a16_gemv_gemm",
    "WEIGHT_GROUP",
    "tint4_pack_weights_groupwise",
    "w4a8_gemm_groupwise",
    "convrot_w4a8_linear_groupwise",
    "tint4_debug_int32_gemm",
    "tint4_debug_w4a8_gemm_even_odd",
    "even_odd_codes",
    "tint4_debug_bounded_wait",
    "tint4_get_device_error",
    "tint4_set_wait_limit_ns",
    "tint4_set_decode_weight_prefetch",
    "tint4_abi_version",
    "QuantizedLinear",
    "GroupwiseQuantizedLinear",
]


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(device: torch.device):
    return torch.cuda.current_stream(device).cuda_stream


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def tint4_abi_version() -> int:
    return int(_native.raw("tint4_abi_version"))


def tint4_pack_weights(W: torch.Tensor, group: int,
                       w_packed: Optional[torch.Tensor] = None,
                       row_scale: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """fp32 W [N, K] -> (packed uint8 [N, K/2], row_scale fp32 [N])."""
    _need(W, "W", torch.float32)
    N, K = W.shape
    if w_packed is None:
        w_packed = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    if row_scale is None:
        row_scale = torch.empty((N,), dtype=torch.float32, device=W.device)
    _need(w_packed, "w_packed", torch.uint8, (N, K // 2))
    _need(row_scale, "row_scale", torch.float32, (N,))
    _native.call("tint4_pack_weights", _ptr(W), N, K, group, _ptr(w_packed), _ptr(row_scale),
                 _stream(W.device))
    return w_packed, row_scale


def convrot_quantize_act(x: torch.Tensor, group: int, bits: int,
                         codes: Optional[torch.Tensor] = None,
                         tok_scale: Optional[torch.Tensor] = None):
    """bf16 x [M, K] -> (codes, tok_scale fp32 [M]); codes int8 [M, K] for
    bits 8, packed uint8 [M, K/2] for bits 4."""
    _need(x, "x", torch.bfloat16)
    M, K = x.shape
    if codes is None:
        codes = (torch.empty((M, K), dtype=torch.int8, device=x.device) if bits == 8 else
                 torch.empty((M, K // 2), dtype=torch.uint8, device=x.device))
    if tok_scale is None:
        tok_scale = torch.empty((M,), dtype=torch.float32, device=x.device)
    if bits == 8:
        _need(codes, "codes", torch.int8, (M, K))
    else:
        _need(codes, "codes", torch.uint8, (M, K // 2))
    _need(tok_scale, "tok_scale", torch.float32, (M,))
    _native.call("convrot_quantize_act", _ptr(x), M, K, group, bits, _ptr(codes),
                 _ptr(tok_scale), _stream(x.device))
    return codes, tok_scale


def _gemm(fn: str, a, tok_scale, w_packed, row_scale, bias, y, a_dtype, a_cols):
    _need(a, "a", a_dtype)
    M = a.shape[0]
    N = w_packed.shape[0]
    K = w_packed.shape[1] * 2
    _need(a, "a", a_dtype, (M, a_cols(K)))
    _need(tok_scale, "tok_scale", torch.float32, (M,))
    _need(w_packed, "w_packed", torch.uint8, (N, K // 2))
    _need(row_scale, "row_scale", torch.float32, (N,))
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, (N,))
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
    _need(y, "y", torch.bfloat16, (M, N))
    _native.call(fn, _ptr(a), _ptr(tok_scale), _ptr(w_packed), _ptr(row_scale), _ptr(bias),
                 _ptr(y), M, N, K, _stream(a.device))
    return y


def w4a8_gemm(a, tok_scale, w_packed, row_scale, bias=None, y=None) -> torch.Tensor:
    """int8 codes a [M, K] x packed int4 W [N, K/2] -> bf16 y [M, N]."""
    return _gemm("w4a8_gemm", a, tok_scale, w_packed, row_scale, bias, y, torch.int8,
                 lambda K: K)


def w4a4_gemm(a_packed, tok_scale, w_packed, row_scale, bias=None, y=None) -> torch.Tensor:
    """packed int4 codes a [M, K/2] x packed int4 W [N, K/2] -> bf16 y [M, N]."""
    return _gemm("w4a4_gemm", a_packed, tok_scale, w_packed, row_scale, bias, y, torch.uint8,
                 lambda K: K // 2)


def w4a4_gemm_widened(a_packed, tok_scale, w_packed, row_scale, bias=None, y=None,
                      workspace=None) -> torch.Tensor:
    """w4a4_gemm whose packed activation codes are widened once into a
    workspace (above 16 tokens) before the int8 tensor-core GEMM: the same
    output bits."""
    _need(a_packed, "a_packed", torch.uint8)
    M = a_packed.shape[0]
    K = 2 * a_packed.shape[1]
    N = w_packed.shape[0]
    _need(tok_scale, "tok_scale", torch.float32, (M,))
    _need(w_packed, "w_packed", torch.uint8, (N, K // 2))
    _need(row_scale, "row_scale", torch.float32, (N,))
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, (N,))
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=a_packed.device)
    _need(y, "y", torch.bfloat16, (M, N))
    need = convrot_linear_workspace_size(M, K, 4)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=a_packed.device)
    _native.call("w4a4_gemm_widened", _ptr(a_packed), _ptr(tok_scale), _ptr(w_packed),
                 _ptr(row_scale), _ptr(bias), _ptr(y), M, N, K, _ptr(workspace), workspace.numel(),
                 _stream(a_packed.device))
    return y


def convrot_linear_workspace_size(M: int, K: int, bits: int) -> int:
    return int(_native.raw("convrot_linear_workspace_size", M, K, bits))


def _linear(fn, bits, x, w_packed, row_scale, group, bias, y, workspace):
    _need(x, "x", torch.bfloat16)
    M, K = x.shape
    N = w_packed.shape[0]
    _need(w_packed, "w_packed", torch.uint8, (N, K // 2))
    _need(row_scale, "row_scale", torch.float32, (N,))
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, (N,))
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _need(y, "y", torch.bfloat16, (M, N))
    need = convrot_linear_workspace_size(M, K, bits)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=x.device)
    _need(workspace, "workspace", torch.uint8)
    _native.call(fn, _ptr(x), _ptr(w_packed), _ptr(row_scale), _ptr(bias), _ptr(y), M, N, K,
                 group, _ptr(workspace), workspace.numel(), _stream(x.device))
    return y


def convrot_w4a8_linear(x, w_packed, row_scale, group, bias=None, y=None, workspace=None):
    """Fused rotate + int8 quantize + W4A8 GEMM: bf16 x [M, K] -> bf16 y [M, N]."""
    return _linear("convrot_w4a8_linear", 8, x, w_packed, row_scale, group, bias, y, workspace)


def convrot_w4a4_linear(x, w_packed, row_scale, group, bias=None, y=None, workspace=None):
    """Fused rotate + int4 quantize + W4A4 GEMM: bf16 x [M, K] -> bf16 y [M, N]."""
    return _linear("convrot_w4a4_linear", 4, x, w_packed, row_scale, group, bias, y, workspace)


def convrot_w4a8_linear_noalloc(x, w_packed, row_scale, group, bias=None, y=None):
    """convrot_w4a8_linear whose scratch is the library's fixed 16 MiB device
    array instead of a caller workspace (for callers that cannot allocate
    device memory).  Calls that overlap on the GPU race on that array."""
    _need(x, "x", torch.bfloat16)
    M, K = x.shape
    N = w_packed.shape[0]
    _need(w_packed, "w_packed", torch.uint8, (N, K // 2))
    _need(row_scale, "row_scale", torch.float32, (N,))
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, (N,))
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _need(y, "y", torch.bfloat16, (M, N))
    _native.call("convrot_w4a8_linear_noalloc", _ptr(x), _ptr(w_packed), _ptr(row_scale),
                 _ptr(bias), _ptr(y), M, N, K, group, _stream(x.device))
    return y


def _scale_dtype(t, name):
    """fp32 scales, or fp16 ones (the pages' stored format): the entry-point
    suffix for that dtype."""
    if t.dtype == torch.float32:
        return ""
    if t.dtype == torch.float16:
        return "_f16"
    raise TypeError(f"{name}: float32 or float16 scales, got {t.dtype}")


def tint4_quantize_weights_int8(W, group: int, w_int8=None, row_scale=None,
                                scale_dtype=torch.float32):
    """fp32 W [N, K] -> rotated int8 codes [N, K] and row scales [N] (W8A8);
    scale_dtype torch.float16 stores the scales in the pages' fp16 format."""
    _need(W, "W", torch.float32)
    N, K = W.shape
    if w_int8 is None:
        w_int8 = torch.empty((N, K), dtype=torch.int8, device=W.device)
    if row_scale is None:
        row_scale = torch.empty((N,), dtype=scale_dtype, device=W.device)
    _need(w_int8, "w_int8", torch.int8, (N, K))
    _need(row_scale, "row_scale", row_scale.dtype, (N,))
    _native.call("tint4_quantize_weights_int8" + _scale_dtype(row_scale, "row_scale"), _ptr(W), N,
                 K, group, _ptr(w_int8), _ptr(row_scale), _stream(W.device))
    return w_int8, row_scale


def w8a8_gemm(a, tok_scale, w_int8, row_scale, bias=None, y=None) -> torch.Tensor:
    """int8 codes a [M, K] x int8 W [N, K] -> bf16 y [M, N]."""
    _need(a, "a", torch.int8)
    M, K = a.shape
    N = w_int8.shape[0]
    _need(tok_scale, "tok_scale", torch.float32, (M,))
    _need(w_int8, "w_int8", torch.int8, (N, K))
    _need(row_scale, "row_scale", row_scale.dtype, (N,))
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, (N,))
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
    _need(y, "y", torch.bfloat16, (M, N))
    _native.call("w8a8_gemm" + _scale_dtype(row_scale, "row_scale"), _ptr(a), _ptr(tok_scale),
                 _ptr(w_int8), _ptr(row_scale), _ptr(bias), _ptr(y), M, N, K, _stream(a.device))
    return y


def convrot_w8a8_linear(x, w_int8, row_scale, group, bias=None, y=None, workspace=None):
    """Fused rotate + int8 quantize + W8A8 GEMM: bf16 x [M, K] -> bf16 y [M, N]."""
    _need(x, "x", torch.bfloat16)
    M, K = x.shape
    N = w_int8.shape[0]
    _need(w_int8, "w_int8", torch.int8, (N, K))
    _need(row_scale, "row_scale", row_scale.dtype, (N,))
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, (N,))
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _need(y, "y", torch.bfloat16, (M, N))
    need = convrot_linear_workspace_size(M, K, 8)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    _native.call("convrot_w8a8_linear" + _scale_dtype(row_scale, "row_scale"), _ptr(x),
                 _ptr(w_int8), _ptr(row_scale), _ptr(bias), _ptr(y), M, N, K, group,
                 _ptr(workspace), workspace.numel(), _stream(x.device))
    return y


def _groups(M, K, device, groups):
    """(w_packed, row_scale, bias or None, y or None) tuples -> ctypes array, ys."""
    if not 1 <= len(groups) <= _native.MAX_GROUPS:
        raise ValueError(f"1 to {_native.MAX_GROUPS} weight groups")
    arr = (_native.WeightGroup * len(groups))()
    ys = []
    for i, (w, sr, bias, y) in enumerate(groups):
        N = w.shape[0]
        _need(w, "w_packed", torch.uint8, (N, K // 2))
        _need(sr, "row_scale", torch.float32, (N,))
        if bias is not None:
            _need(bias, "bias", torch.bfloat16, (N,))
        if y is None:
            y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        _need(y, "y", torch.bfloat16, (M, N))
        arr[i] = _native.WeightGroup(_ptr(w), _ptr(sr), _ptr(bias), _ptr(y), N)
        ys.append(y)
    return arr, ys


def w4a8_gemm_grouped(a, tok_scale, groups):
    """int8 codes a [M, K] times each (w_packed [N_g, K/2], row_scale [N_g],
    bias [N_g] or None, y [M, N_g] or None) of `groups`, one launch for all;
    returns the list of bf16 outputs."""
    _need(a, "a", torch.int8)
    M, K = a.shape
    _need(tok_scale, "tok_scale", torch.float32, (M,))
    arr, ys = _groups(M, K, a.device, groups)
    _native.call("w4a8_gemm_grouped", _ptr(a), _ptr(tok_scale), ctypes.addressof(arr),
                 len(groups), M, K, _stream(a.device))
    return ys


def convrot_w4a8_linear_grouped(x, groups, group, workspace=None):
    """Rotate + int8 quantize x once, then w4a8_gemm_grouped over `groups`."""
    _need(x, "x", torch.bfloat16)
    M, K = x.shape
    arr, ys = _groups(M, K, x.device, groups)
    need = convrot_linear_workspace_size(M, K, 8)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    _native.call("convrot_w4a8_linear_grouped", _ptr(x), ctypes.addressof(arr), len(groups),
                 M, K, group, _ptr(workspace), workspace.numel(), _stream(x.device))
    return ys


def w4a16_gemv_gemm(x, w_q, scale, zero, group: int = 128, y=None) -> torch.Tensor:
    """bf16 x [M, K], uint4 w_q [N, K/2], bf16 scale / uint8 zero [N, K/group]
    -> bf16 y [M, N]."""
    _need(x, "x", torch.bfloat16)
    M, K = x.shape
    N = w_q.shape[0]
    _need(w_q, "w_q", torch.uint8, (N, K // 2))
    _need(scale, "scale", torch.bfloat16, (N, K // group))
    _need(zero, "zero", torch.uint8, (N, K // group))
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _need(y, "y", torch.bfloat16, (M, N))
    _native.call("w4a16_gemv_gemm", _ptr(x), _ptr(w_q), _ptr(scale), _ptr(zero), group, _ptr(y),
                 M, N, K, _stream(x.device))
    return y


def tint4_debug_int32_gemm(a, act_bits: int, w_packed, acc=None) -> torch.Tensor:
    """Raw int32 accumulators of the tensor-core GEMM (tests)."""
    M = a.shape[0]
    N = w_packed.shape[0]
    K = w_packed.shape[1] * 2
    _need(a, "a", torch.int8 if act_bits == 8 else torch.uint8,
          (M, K if act_bits == 8 else K // 2))
    _need(w_packed, "w_packed", torch.uint8, (N, K // 2))
    if acc is None:
        acc = torch.empty((M, N), dtype=torch.int32, device=a.device)
    _need(acc, "acc", torch.int32, (M, N))
    _native.call("tint4_debug_int32_gemm", _ptr(a), act_bits, _ptr(w_packed), _ptr(acc), M, N, K,
                 _stream(a.device))
    return acc


WEIGHT_GROUP = 128   # K values per group-wise weight scale (TINT4_WEIGHT_GROUP)


def tint4_pack_weights_groupwise(W: torch.Tensor, group: int, asym: bool = False,
                                 w_packed=None, w_scale=None, w_zero=None,
                                 scale_dtype=torch.float32):
    """fp32 W [N, K] -> (packed uint8 [N, K/2], scale [N, K/128], zero uint8
    [N, K/128] or None): rotated, then int4 per 128-wide K group (symmetric,
    or asymmetric with zero points).  scale_dtype torch.float16 stores the
    scales in the pages' fp16 format (codes taken against the fp16 scale)."""
    _need(W, "W", torch.float32)
    N, K = W.shape
    ng = K // WEIGHT_GROUP
    if w_packed is None:
        w_packed = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    if w_scale is None:
        w_scale = torch.empty((N, ng), dtype=scale_dtype, device=W.device)
    if asym and w_zero is None:
        w_zero = torch.empty((N, ng), dtype=torch.uint8, device=W.device)
    _need(w_packed, "w_packed", torch.uint8, (N, K // 2))
    _need(w_scale, "w_scale", w_scale.dtype, (N, ng))
    if asym:
        _need(w_zero, "w_zero", torch.uint8, (N, ng))
    _native.call("tint4_pack_weights_groupwise" + _scale_dtype(w_scale, "w_scale"), _ptr(W), N, K,
                 group, int(bool(asym)), _ptr(w_packed), _ptr(w_scale),
                 _ptr(w_zero if asym else None), _stream(W.device))
    return w_packed, w_scale, (w_zero if asym else None)


def _gw_operands(M, K, w_packed, w_scale, w_zero, bias, y, device):
    N = w_packed.shape[0]
    ng = K // WEIGHT_GROUP
    _need(w_packed, "w_packed", torch.uint8, (N, K // 2))
    _need(w_scale, "w_scale", w_scale.dtype, (N, ng))
    _scale_dtype(w_scale, "w_scale")
    if w_zero is not None:
        _need(w_zero, "w_zero", torch.uint8, (N, ng))
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, (N,))
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
    _need(y, "y", torch.bfloat16, (M, N))
    return N, y


def w4a8_gemm_groupwise(a, tok_scale, w_packed, w_scale, w_zero=None, bias=None,
                        y=None) -> torch.Tensor:
    """int8 codes a [M, K] x group-wise packed int4 W [N, K/2] -> bf16 y [M, N]."""
    _need(a, "a", torch.int8)
    M, K = a.shape
    _need(tok_scale, "tok_scale", torch.float32, (M,))
    N, y = _gw_operands(M, K, w_packed, w_scale, w_zero, bias, y, a.device)
    _native.call("w4a8_gemm_groupwise" + _scale_dtype(w_scale, "w_scale"), _ptr(a),
                 _ptr(tok_scale), _ptr(w_packed), _ptr(w_scale), _ptr(w_zero), _ptr(bias), _ptr(y),
                 M, N, K, _stream(a.device))
    return y


def convrot_w4a8_linear_groupwise(x, w_packed, w_scale, group, w_zero=None, bias=None, y=None,
                                  workspace=None) -> torch.Tensor:
    """Fused rotate + int8 quantize + group-wise W4A8 GEMM: bf16 x [M, K] -> y."""
    _need(x, "x", torch.bfloat16)
    M, K = x.shape
    N, y = _gw_operands(M, K, w_packed, w_scale, w_zero, bias, y, x.device)
    need = convrot_linear_workspace_size(M, K, 8)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    _native.call("convrot_w4a8_linear_groupwise" + _scale_dtype(w_scale, "w_scale"), _ptr(x),
                 _ptr(w_packed), _ptr(w_scale), _ptr(w_zero), _ptr(bias), _ptr(y), M, N, K, group,
                 _ptr(workspace), workspace.numel(), _stream(x.device))
    return y


def even_odd_codes(codes: torch.Tensor) -> torch.Tensor:
    """int8 codes [M, K] in natural K order -> the even/odd K order of
    tint4_debug_w4a8_gemm_even_odd (positions 0, 2, 4, 6, 1, 3, 5, 7 of every
    block of 8).  A layout change only (torch ops, test and timing set-up)."""
    M, K = codes.shape
    return codes.view(M, K // 8, 4, 2).transpose(2, 3).contiguous().view(M, K)


def tint4_debug_w4a8_gemm_even_odd(a_even_odd, tok_scale, w_packed, row_scale, bias=None,
                                   y=None) -> torch.Tensor:
    """The fused linears' GEMM launch (M > 16) on even/odd-order int8 codes."""
    return _gemm("tint4_debug_w4a8_gemm_even_odd", a_even_odd, tok_scale, w_packed, row_scale,
                 bias, y, torch.int8, lambda K: K)


def tint4_debug_bounded_wait(limit_ns: int, device=None) -> None:
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    _native.call("tint4_debug_bounded_wait", int(limit_ns), _stream(dev))


def tint4_get_device_error(device=None) -> int:
    """Synchronize the current stream, then read + clear the device error word.
    Returns the raw status (0 = ok, 5 = a bounded wait gave up)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    return int(_native.raw("tint4_get_device_error", _stream(dev)))


def tint4_set_wait_limit_ns(limit_ns: int) -> None:
    _native.call("tint4_set_wait_limit_ns", int(limit_ns))


def tint4_set_decode_weight_prefetch(enable: bool) -> None:
    """Let the small-M kernels stream their weights before the previous kernel
    of the stream has finished (see the header: only when that kernel does not
    write the weights).  Process-wide; off by default."""
    _native.call("tint4_set_decode_weight_prefetch", 1 if enable else 0)


class QuantizedLinear:
    """A W4A8 / W4A4 ConvRot linear layer holding its packed weights.

    The layer form the pages use ("ComfyUI-INT-Crush", "Forward Pass"): the
    weights are rotated, quantized and packed once (``from_float``); each call
    rotates + quantizes the activations and runs the integer GEMM."""

    def __init__(self, w_packed, row_scale, group: int, act_bits: int = 8, bias=None):
        self.w_packed = w_packed
        self.row_scale = row_scale
        self.group = group
        self.act_bits = act_bits
        self.bias = bias
        self._workspace = None

    @classmethod
    def from_float(cls, W: torch.Tensor, group: int, act_bits: int = 8, bias=None):
        wp, sr = tint4_pack_weights(W.float().contiguous(), group)
        return cls(wp, sr, group, act_bits, bias)

    @property
    def out_features(self) -> int:
        return self.w_packed.shape[0]

    @property
    def in_features(self) -> int:
        return self.w_packed.shape[1] * 2

    def __call__(self, x: torch.Tensor, y: Optional[torch.Tensor] = None) -> torch.Tensor:
        M = x.shape[0]
        need = convrot_linear_workspace_size(M, self.in_features, self.act_bits)
        if self._workspace is None or self._workspace.numel() < need or \
                self._workspace.device != x.device:
            self._workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=x.device)
        fn = convrot_w4a8_linear if self.act_bits == 8 else convrot_w4a4_linear
        return fn(x, self.w_packed, self.row_scale, self.group, self.bias, y, self._workspace)


class GroupwiseQuantizedLinear:
    """A W4A8 ConvRot linear layer with group-wise weight scales (one per row
    and 128-wide K group; symmetric, or asymmetric with zero points).

    "ComfyUI-INT-Crush", "Weight Format" (scales [out, num_groups]) and
    "feat: packed int4 convrot model loading and dispatch", "Summary" (the
    asymmetric W4A8 format): the weights are rotated and quantized once
    (``from_float``); each call rotates + quantizes the activations to int8
    and runs the group-wise GEMM."""

    def __init__(self, w_packed, w_scale, w_zero, group: int, bias=None):
        self.w_packed = w_packed
        self.w_scale = w_scale
        self.w_zero = w_zero
        self.group = group
        self.bias = bias
        self._workspace = None

    @classmethod
    def from_float(cls, W: torch.Tensor, group: int, asym: bool = False, bias=None,
                   scale_dtype=torch.float32):
        wp, s, z = tint4_pack_weights_groupwise(W.float().contiguous(), group, asym,
                                                scale_dtype=scale_dtype)
        return cls(wp, s, z, group, bias)

    @property
    def out_features(self) -> int:
        return self.w_packed.shape[0]

    @property
    def in_features(self) -> int:
        return self.w_packed.shape[1] * 2

    def __call__(self, x: torch.Tensor, y: Optional[torch.Tensor] = None) -> torch.Tensor:
        need = convrot_linear_workspace_size(x.shape[0], self.in_features, 8)
        if self._workspace is None or self._workspace.numel() < need or \
                self._workspace.device != x.device:
            self._workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=x.device)
        return convrot_w4a8_linear_groupwise(x, self.w_packed, self.w_scale, self.group,
                                             self.w_zero, self.bias, y, self._workspace)
