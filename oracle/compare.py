"""Comparison of a bf16 result with the oracle (TEST INFRASTRUCTURE ONLY).

The layer's outputs are bf16.  The oracle evaluates each output in fp64 and
rounds it once; the kernel evaluates it in fp32 and rounds it once.  Where the
exact value lies within the fp32 evaluation error of a bf16 rounding midpoint,
both neighbours are correct roundings of a valid evaluation, and the two sides
may pick different ones: a one-ulp difference that can land on an element of
any size.  Such elements are rounding ties, the analogue of the activation
codes' ties: they must be rare and exactly one ulp apart.  Every other element
is held to the layer's tolerance, max |gpu - oracle| / rms(oracle) <= 1e-2.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import bf16_bits_to_f32, round_bf16, w4a16_weights_f64

Y_TOL = 1e-2          # max |gpu - oracle| / rms(oracle) outside ties
# At most this fraction of outputs may be rounding ties.  An fp32 evaluation
# with relative error e disagrees with the exact rounding on about
# 2 e / 2^-8 of the outputs: e ~ 2^-23 for the integer GEMM's epilogue (two
# or three fp32 roundings of an exact int32 sum) gives ~6e-5, bounded here by
# 1e-3.  Kernels whose error bound is given per element (W4A16: tensor-core
# dot products) pass the fraction that bound allows instead (tie_capacity).
TIE_FRAC = 1e-3


def bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _order_key(b: np.ndarray) -> np.ndarray:
    """bf16 bits -> integers ordered like the values (adjacent values differ by 1)."""
    b = np.asarray(b, np.uint16).astype(np.int64)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


@dataclass
class Bf16Check:
    max_rel: float        # max |gpu - oracle| / rms(oracle) over non-tie elements
    ties: int             # one-ulp differences at rounding midpoints
    n: int
    worst_index: int
    tie_limit: float = TIE_FRAC

    @property
    def tie_frac(self) -> float:
        return self.ties / max(self.n, 1)

    @property
    def ok(self) -> bool:
        return self.max_rel <= Y_TOL and self.tie_frac <= self.tie_limit

    def __str__(self):
        return (f"max|diff|/rms={self.max_rel:.3e} (tol {Y_TOL}), ties={self.ties}/{self.n} "
                f"(<= {self.tie_limit:g}), worst at {self.worst_index}")


def check_bf16(gpu_bits: np.ndarray, ref_f64: np.ndarray, err_abs,
               tie_limit: float = TIE_FRAC) -> Bf16Check:
    """Compare bf16 results (bits) with the oracle's unrounded fp64 values.

    err_abs: bound (scalar or per element) on the fp32 evaluation error of
    the value before its bf16 rounding, or a function of flat indices that
    returns the bound of those elements (only the elements whose roundings
    differ need it)."""
    ref_arr = np.asarray(ref_f64, np.float64)
    g_bits = np.asarray(gpu_bits, np.uint16).ravel()
    ref = ref_arr.ravel()
    o_bits = round_bf16(ref)
    g = bits_to_f64(g_bits)
    o = bits_to_f64(o_bits)
    rms = float(np.sqrt(np.mean(o ** 2))) if o.size else 0.0
    # only the elements whose roundings differ can be ties or errors
    idx = np.flatnonzero(g_bits != o_bits)
    adjacent = np.abs(_order_key(g_bits[idx]) - _order_key(o_bits[idx])) == 1
    gi, oi = g[idx], o[idx]
    if callable(err_abs):
        err_i = np.asarray(err_abs(idx), np.float64)
    else:
        err_i = np.broadcast_to(np.asarray(err_abs, np.float64), ref_arr.shape).ravel()[idx]
    tie = adjacent & (np.abs(ref[idx] - 0.5 * (gi + oi)) <= err_i)
    d = np.where(tie, 0.0, np.abs(gi - oi))
    if d.size:
        j = int(np.argmax(d))
        worst, dmax = int(idx[j]), float(d[j])
    else:
        worst, dmax = (0 if ref.size else -1), 0.0
    max_rel = dmax / rms if rms > 0 else dmax
    return Bf16Check(max_rel=max_rel, ties=int(tie.sum()), n=int(ref.size), worst_index=worst,
                     tie_limit=tie_limit)


def gemm_eval_error(ref_f64: np.ndarray, bias_f64=None) -> np.ndarray:
    """fp32 evaluation error bound of acc * s_tok * s_row (+ bias): two or
    three roundings of at most 2^-24 relative each, bounded by 2^-20 of the
    magnitudes involved."""
    mag = np.abs(np.asarray(ref_f64, np.float64))
    if bias_f64 is not None:
        mag = mag + np.abs(np.asarray(bias_f64, np.float64))
    return mag * 2.0 ** -20


# --------------------------------------------------------------------------
# W4A16: per-element bounds of the kernels' fp32 evaluation
# --------------------------------------------------------------------------
#
# Model of the tensor cores' fp32 accumulation (warp-level mma.m16n8k16 and
# tcgen05.mma kind::f16): the products of bf16 operands are exact in fp32; one
# instruction adds its 16 products per output to the accumulator with at most
# two roundings of at most 2^-23 relative to the magnitudes involved (the
# adder's alignment and rounding).  A chain of c such instructions on one
# output is then off by at most c 2^-22 sum |terms|.  Scalar fp32 fma/add:
# one rounding of 2^-24 relative.  The bounds are magnitudes of terms, so they
# come from |x| @ |w|^T products (a library matrix product on the oracle's
# weights).


def _abs_x(x_bits) -> np.ndarray:
    return np.abs(bf16_bits_to_f32(x_bits).astype(np.float64))


def w4a16_stream_error(x_bits, q_packed, scale_bits, zero, group) -> np.ndarray:
    """Bound [M, N] on |kernel - exact| before the output rounding for the
    streaming W4A16 kernel (up to 32 tokens).  Per group j of `group` = 128
    values it forms s_j (S1 - (128 + z_j) S2) with S1 = sum x (128 + q) and
    S2 = sum x, each a chain of 8 k16 MMAs, so the MMAs are off by at most
    8 2^-22 s_j (sum |x| (128 + q) + (128 + z_j) sum |x|); then one fma per
    group for the difference and one per group for the running sum, and up
    to 16 warp partial sums added at the end: (K / group + 18) 2^-24 of
    sum |x| |w|, w = (q - z) s."""
    xa = _abs_x(x_bits)
    K = xa.shape[1]
    w = w4a16_weights_f64(q_packed, scale_bits, zero, group)
    q = np.asarray(q_packed, np.uint8)
    qk = np.empty((q.shape[0], K), np.float64)
    qk[:, 0::2] = q & 0xF
    qk[:, 1::2] = q >> 4
    zk = np.repeat(np.asarray(zero, np.float64), group, axis=1)
    sk = np.repeat(bf16_bits_to_f32(scale_bits).astype(np.float64), group, axis=1)
    w_off = sk * (256.0 + qk + zk)
    return 8 * 2.0 ** -22 * (xa @ w_off.T) + (K // group + 18) * 2.0 ** -24 * (xa @ np.abs(w).T)


def w4a16_tc_error(x_bits, w_widened: np.ndarray) -> np.ndarray:
    """Bound [M, N] on |kernel - 16-bit unpack form| before the output
    rounding for the tcgen05 W4A16 GEMM (above 32 tokens): one chain of K / 16
    MMAs on bf16 operands, (K / 16 + 1) 2^-22 sum |x| |w_bf16|."""
    xa = _abs_x(x_bits)
    K = xa.shape[1]
    return (K // 16 + 1) * 2.0 ** -22 * (xa @ np.abs(w_widened).T)


def tie_capacity(ref_f64: np.ndarray, err) -> float:
    """Fraction of elements whose value lies within err (per element) of a
    bf16 rounding midpoint: the only elements a kernel within that error
    bound may round to the other neighbour.  With a per-element bound this is
    the tie budget the arithmetic gives."""
    ref = np.asarray(ref_f64, np.float64).ravel()
    if ref.size == 0:
        return 0.0
    e = np.broadcast_to(np.asarray(err, np.float64), np.asarray(ref_f64).shape).ravel()
    o = bits_to_f64(round_bf16(ref))
    a = np.abs(o)
    expo = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    ulp = np.where(a > 0, 2.0 ** (expo - 7), 2.0 ** -133)
    # at a power of two the spacing below is half the spacing above
    pow2 = a == 2.0 ** expo
    ulp = np.where(pow2 & (np.abs(ref) < a), ulp / 2, ulp)
    dist = ulp / 2 - np.abs(ref - o)
    return float(np.count_nonzero(dist <= e)) / ref.size
