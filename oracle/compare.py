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

from . import round_bf16

Y_TOL = 1e-2          # max |gpu - oracle| / rms(oracle) outside ties
# At most this fraction of outputs may be rounding ties.  An fp32 evaluation
# with relative error e disagrees with the exact rounding on about
# 2 e / 2^-8 of the outputs: e ~ 2^-23 for the integer GEMM's epilogue (two
# or three fp32 roundings of an exact int32 sum) gives ~6e-5, bounded here by
# 1e-3; e ~ 1e-5 for fp32 dot products of K = 4096 summed on the tensor cores
# gives ~5e-3, the bound the W4A16 tests pass explicitly.
TIE_FRAC = 1e-3
TIE_FRAC_ACCUMULATED = 5e-3


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
    the value before its bf16 rounding."""
    ref_arr = np.asarray(ref_f64, np.float64)
    g_bits = np.asarray(gpu_bits, np.uint16).ravel()
    ref = ref_arr.ravel()
    o_bits = round_bf16(ref)
    g = bits_to_f64(g_bits)
    o = bits_to_f64(o_bits)
    err = np.broadcast_to(np.asarray(err_abs, np.float64), ref_arr.shape).ravel()
    differ = g_bits != o_bits
    adjacent = np.abs(_order_key(g_bits) - _order_key(o_bits)) == 1
    tie = differ & adjacent & (np.abs(ref - 0.5 * (g + o)) <= err)
    rms = float(np.sqrt(np.mean(o ** 2))) if o.size else 0.0
    d = np.where(tie, 0.0, np.abs(g - o))
    worst = int(np.argmax(d)) if d.size else -1
    dmax = float(d.max()) if d.size else 0.0
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


def accumulation_error(ref_f64: np.ndarray, rel: float = 1e-4) -> float:
    """Bound used for fp32 dot products summed in an order the oracle does not
    follow (tensor-core accumulation): rel * rms of the result."""
    r = np.asarray(ref_f64, np.float64)
    return rel * float(np.sqrt(np.mean(r ** 2))) if r.size else 0.0
