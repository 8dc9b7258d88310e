"""Helpers shared by the GPU tests: numpy <-> torch transfers and the
tolerances the parity tests apply."""
import numpy as np
import torch

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


def code_mismatch(gpu_codes: np.ndarray, ref_codes: np.ndarray):
    """(fraction of differing codes, max |difference|)."""
    d = np.abs(gpu_codes.astype(np.int32) - ref_codes.astype(np.int32))
    return float(np.count_nonzero(d)) / d.size, int(d.max()) if d.size else 0
