"""Seeded synthetic inputs for the quantized linear layer.

This module only draws random numbers and lays them out: it holds none of the
layer's arithmetic (no rotation, no quantization, no packing of codes), so the
tests can feed the very same inputs to the CUDA path and to the CPU oracle.

The value distributions follow the diffusion-transformer workloads the pages
run (FLUX.2-klein and Z-Image inference in "feat: packed int4 convrot model
loading and dispatch", section "Verification"; their weights are not
available, so seeded synthetic tensors of the same shapes stand in):

* activations: bf16, N(0, 1), with a fixed set of outlier channels scaled up
  (ceil(1% of K) channels x50 for the attention projections, ceil(0.5% of K)
  channels x30 on a GELU input for the MLP down projection) -- the outlier
  structure that makes the Hadamard rotation worthwhile ("TINT4 v1.2",
  "量化方案": QuaRot is advised when the outlier score is high);
* weights to be quantized: fp32 N(0, 0.02);
* W4A16 operands: uint4 codes and zero points uniform on 0..15 (two random
  nibbles per byte), bf16 scales |N(0, 0.02)| / 8 + 1e-4.

Every array is a numpy array; bf16 tensors are returned as their uint16 bit
patterns.  The default seed is 42, the seed of the pages' own runs.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

SEED = 42


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([seed, stream]))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (torch's round-to-nearest-even cast)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def outlier_channels(K: int, frac: float, seed: int = SEED, stream: int = 7) -> np.ndarray:
    """A fixed, seeded set of ceil(frac * K) channel indices (shared by all tokens)."""
    n = max(1, math.ceil(frac * K))
    return np.sort(_rng(seed, stream).choice(K, size=n, replace=False))


def activations(M: int, K: int, seed: int = SEED, outlier_frac: float = 0.01,
                outlier_gain: float = 50.0, stream: int = 1) -> np.ndarray:
    """x bf16 [M, K]: N(0, 1) with ceil(outlier_frac*K) channels x outlier_gain."""
    x = _rng(seed, stream).standard_normal((M, K), dtype=np.float32)
    if outlier_frac > 0:
        x[:, outlier_channels(K, outlier_frac, seed)] *= np.float32(outlier_gain)
    return f32_to_bf16_bits(x)


def gelu_activations(M: int, K: int, seed: int = SEED, outlier_frac: float = 0.005,
                     outlier_gain: float = 30.0, stream: int = 2) -> np.ndarray:
    """MLP down-projection input: GELU (erf form) of N(0, 1), then
    ceil(outlier_frac*K) channels x outlier_gain, rounded to bf16."""
    z = _rng(seed, stream).standard_normal((M, K), dtype=np.float32)
    t = torch.from_numpy(z)
    g = torch.nn.functional.gelu(t, approximate="none").numpy()
    if outlier_frac > 0:
        g[:, outlier_channels(K, outlier_frac, seed, stream=8)] *= np.float32(outlier_gain)
    return f32_to_bf16_bits(g)


def weights(N: int, K: int, seed: int = SEED, std: float = 0.02, stream: int = 3) -> np.ndarray:
    """W fp32 [N, K] ~ N(0, std)."""
    return (_rng(seed, stream).standard_normal((N, K), dtype=np.float32) * np.float32(std))


@dataclass
class W4A16Operands:
    x: np.ndarray        # bf16 bits [M, K]
    q: np.ndarray        # uint8 [N, K/2], two uint4 codes per byte
    scale: np.ndarray    # bf16 bits [N, K/group]
    zero: np.ndarray     # uint8 [N, K/group], values 0..15
    group: int


def w4a16_operands(M: int, N: int, K: int, group: int = 128, seed: int = SEED,
                   stream: int = 4) -> W4A16Operands:
    """Operands of the W4A16 group-wise asymmetric layer (torchao-style triple)."""
    r = _rng(seed, stream)
    x = f32_to_bf16_bits(r.standard_normal((M, K), dtype=np.float32))
    q = r.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    zero = r.integers(0, 16, size=(N, K // group), dtype=np.uint8)
    s = np.abs(r.standard_normal((N, K // group), dtype=np.float32)) * np.float32(0.02 / 8.0)
    scale = f32_to_bf16_bits(s + np.float32(1e-4))
    return W4A16Operands(x=x, q=q, scale=scale, zero=zero, group=group)


def random_codes(rows: int, K: int, lo: int, hi: int, seed: int = SEED,
                 stream: int = 5) -> np.ndarray:
    """Uniform integer codes in [lo, hi] as int8 [rows, K] (for GEMM-only tests)."""
    return _rng(seed, stream).integers(lo, hi + 1, size=(rows, K), dtype=np.int8)


def random_bytes(rows: int, cols: int, seed: int = SEED, stream: int = 6) -> np.ndarray:
    """Uniform random bytes uint8 [rows, cols] (random packed nibble pairs)."""
    return _rng(seed, stream).integers(0, 256, size=(rows, cols), dtype=np.uint8)


def positive_scales(n: int, seed: int = SEED, stream: int = 9, lo: float = 1e-3,
                    hi: float = 1e-1) -> np.ndarray:
    """fp32 [n] log-uniform positive scales (for GEMM-only tests)."""
    r = _rng(seed, stream)
    return np.exp(r.uniform(np.log(lo), np.log(hi), size=n)).astype(np.float32)


# ---------------------------------------------------------------------------
# Named workloads (the shapes of the pages' diffusion-transformer layers)
# ---------------------------------------------------------------------------

WORKLOADS = {
    # tiny ConvRot W4A8 linear
    "tiny_w4a8": dict(M=64, K=256, N=256, group=256, act_bits=8, x="attn"),
    # fused-QKV attention projection: 64x64 latent patches + 512 text tokens
    "dit_qkv_w4a8": dict(M=4608, K=3072, N=9216, group=256, act_bits=8, x="attn"),
    "dit_qkv_w4a4": dict(M=4608, K=3072, N=9216, group=256, act_bits=4, x="attn"),
    # the same layer with group-wise asymmetric weights (scale + zero point per
    # row and 128-wide K group)
    "dit_qkv_w4a8_asym_g128": dict(M=4608, K=3072, N=9216, group=256, act_bits=8, x="attn",
                                   weight_group=128, asym=True),
    # MLP pair, group 64
    "dit_mlp_up_w4a8": dict(M=4608, K=3072, N=12288, group=64, act_bits=8, x="attn"),
    "dit_mlp_down_w4a8": dict(M=4608, K=12288, N=3072, group=64, act_bits=8, x="gelu"),
    # small-M text-encoder decode
    "te_decode_w4a16": dict(Ms=(1, 4, 16), K=4096, N=12288, group=128),
    # the same layer on a prefill batch: the tensor-core branch
    "te_prefill_w4a16": dict(M=4096, K=4096, N=12288, group=128),
    "te_decode_w4a8": dict(Ms=(1, 4, 16), K=4096, N=12288, group=256, act_bits=8, x="attn"),
}


def layer_inputs(name: str, seed: int = SEED, M: int | None = None):
    """(x bf16 bits [M, K], W fp32 [N, K]) for one named W4A8/W4A4 workload."""
    w = WORKLOADS[name]
    M = M if M is not None else w["M"]
    if w.get("x") == "gelu":
        x = gelu_activations(M, w["K"], seed)
    else:
        x = activations(M, w["K"], seed)
    return x, weights(w["N"], w["K"], seed)
