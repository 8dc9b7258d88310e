"""Column-parallel (N-split) sharding of the quantized linear across ranks.

y = x W^T splits along N with no exchange: every output column y[:, n] is
computed from x and weight row n alone (its row scale, its packed nibbles,
the token scales of x), so rank r of G holds the weight rows [lo_r, hi_r)
and their row scales, receives the whole x, and writes y[:, lo_r:hi_r] with
the same bits the unsharded layer gives those columns.  An optional
all-gather assembles the full y on every rank (NCCL over NVLink / NVSwitch
between GPUs; any torch.distributed backend works).

The shard boundaries are multiples of 16 (the GEMM's row-block rule), as
equal as that allows; the last shard may be narrower.  The compute of a
shard is the library's fused linear (convrot_w4a8_linear or
convrot_w4a4_linear) unless a caller passes its own `linear` (the CPU tests
do, to check the host logic without a GPU).
"""
from __future__ import annotations

from typing import Callable, List, Optional, Tuple

import torch
import torch.distributed as dist

ROW_ALIGN = 16


def shard_bounds(N: int, world: int, align: int = ROW_ALIGN) -> List[Tuple[int, int]]:
    """[lo, hi) weight rows of each of `world` ranks: contiguous, disjoint,
    covering [0, N), every boundary a multiple of `align` (N itself may not
    be), widths as equal as that allows (the first shards are the wider)."""
    if N < 0 or world < 1 or align < 1:
        raise ValueError("N >= 0, world >= 1, align >= 1")
    blocks = (N + align - 1) // align
    q, r = divmod(blocks, world)
    bounds, lo = [], 0
    for i in range(world):
        hi = min(N, lo + (q + (1 if i < r else 0)) * align)
        bounds.append((lo, hi))
        lo = hi
    return bounds


class ColumnParallelLinear:
    """One rank's shard of a ConvRot W4A8 / W4A4 linear layer.

    w_packed [N_r, K/2] and row_scale [N_r] are this rank's rows (rows
    [lo, hi) of the full layer; ``shard`` slices them out of a packed full
    layer).  ``__call__(x)`` returns y[:, lo:hi] [M, N_r], or with
    gather=True the full y [M, N] assembled from every rank's shard."""

    def __init__(self, w_packed: torch.Tensor, row_scale: torch.Tensor, group: int, N: int,
                 rank: int, world: int, act_bits: int = 8, bias: Optional[torch.Tensor] = None,
                 gather: bool = False, process_group=None,
                 linear: Optional[Callable] = None):
        self.bounds = shard_bounds(N, world)
        self.lo, self.hi = self.bounds[rank]
        if w_packed.shape[0] != self.hi - self.lo or row_scale.shape[0] != self.hi - self.lo:
            raise ValueError(f"rank {rank} holds rows [{self.lo}, {self.hi}): got "
                             f"{w_packed.shape[0]} packed rows, {row_scale.shape[0]} scales")
        self.w_packed, self.row_scale = w_packed, row_scale
        self.bias = bias
        self.group, self.N, self.rank, self.world = group, N, rank, world
        self.act_bits = act_bits
        self.gather = gather
        self.pg = process_group
        if linear is None:
            from . import convrot_w4a4_linear, convrot_w4a8_linear
            linear = convrot_w4a8_linear if act_bits == 8 else convrot_w4a4_linear
        self._linear = linear

    @staticmethod
    def shard(full_w_packed: torch.Tensor, full_row_scale: torch.Tensor, rank: int, world: int,
              full_bias: Optional[torch.Tensor] = None):
        """This rank's rows of a packed full layer (a row of the packed
        matrix is one weight row: the rotation and the nibbles run along K)."""
        lo, hi = shard_bounds(full_w_packed.shape[0], world)[rank]
        bias = None if full_bias is None else full_bias[lo:hi].contiguous()
        return full_w_packed[lo:hi].contiguous(), full_row_scale[lo:hi].contiguous(), bias

    def __call__(self, x: torch.Tensor, workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
        if self.hi > self.lo:
            y_local = self._linear(x, self.w_packed, self.row_scale, self.group, self.bias, None,
                                   workspace)
        else:
            y_local = torch.empty((x.shape[0], 0), dtype=torch.bfloat16, device=x.device)
        if not self.gather:
            return y_local
        return self.assemble(y_local)

    def assemble(self, y_local: torch.Tensor) -> torch.Tensor:
        """All-gather the ranks' column shards into y [M, N]: shards are padded
        to the widest one for the collective, then placed at their columns."""
        M = y_local.shape[0]
        width = max(hi - lo for lo, hi in self.bounds)
        pad = torch.zeros((M, width), dtype=y_local.dtype, device=y_local.device)
        pad[:, : y_local.shape[1]] = y_local
        # the collective moves bytes (every backend has uint8; not all have bf16)
        raw = pad.view(torch.uint8)
        parts = [torch.empty_like(raw) for _ in range(self.world)]
        dist.all_gather(parts, raw, group=self.pg)
        y = torch.empty((M, self.N), dtype=y_local.dtype, device=y_local.device)
        for (lo, hi), p in zip(self.bounds, parts):
            y[:, lo:hi] = p.view(y_local.dtype)[:, : hi - lo]
        return y
