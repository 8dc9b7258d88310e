"""Helpers shared by the GPU tests: numpy <-> torch transfers and the
tolerances the parity tests apply."""
import numpy as np
import torch

# bf16 outputs: max |gpu - oracle| / rms(oracle) must stay within this.
Y_TOL = 1e-2
# activation codes may differ from the oracle only at rounding ties: at most
# this fraction of elements, each by at most 1.
CODE_MISMATCH_FRAC = 1e-4


def dev():
    return torch.device("cuda", 0)


def to_gpu(a: np.ndarray, dtype=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.to(dev())


def bf16_to_gpu(bits: np.ndarray) -> torch.Tensor:
    return to_gpu(np.ascontiguousarray(bits).view(np.int16), torch.bfloat16)


def bf16_from_gpu(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rel_err(gpu_bits: np.ndarray, ref_bits: np.ndarray) -> float:
    g = bits_to_f64(gpu_bits)
    r = bits_to_f64(ref_bits)
    rms = np.sqrt(np.mean(r ** 2))
    if rms == 0:
        return float(np.abs(g - r).max())
    return float(np.abs(g - r).max() / rms)


def code_mismatch(gpu_codes: np.ndarray, ref_codes: np.ndarray):
    """(fraction of differing codes, max |difference|)."""
    d = np.abs(gpu_codes.astype(np.int32) - ref_codes.astype(np.int32))
    return float(np.count_nonzero(d)) / d.size, int(d.max()) if d.size else 0
