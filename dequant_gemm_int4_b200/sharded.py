"""An Int4 linear layer whose weight rows are split across the ranks of a
process group (one process per GPU).

Quantization, packing and the matmul are independent per weight row: row n
of W has its own groups, scales and codes, and output column n of y depends
only on row n.  So each rank holds the rows [start, stop) that shard_rows
assigns it (packed codes, scales, zero points and bias of those rows; the
slices of a whole-matrix quantization, bit for bit), computes its output
columns with the library's fused matmul, and one all-gather over the group
assembles y [M, N] on every rank.  x is replicated.  The collective is
torch.distributed's (NCCL over NVLink on GPUs, gloo on CPU).
"""

from __future__ import annotations

from typing import Callable

import torch
import torch.distributed as dist

__all__ = ["shard_rows", "shard_quantized", "ShardedInt4Linear"]


def shard_rows(N: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [start, stop) of rank `rank`: contiguous, sizes differing by at
    most one, the larger shards first."""
    if world < 1 or not 0 <= rank < world or N < 0:
        raise ValueError("need world >= 1, 0 <= rank < world and N >= 0")
    base, rem = divmod(N, world)
    start = rank * base + min(rank, rem)
    return start, start + base + (1 if rank < rem else 0)


def shard_quantized(packed, scales, zeros, bias, world: int, rank: int):
    """This rank's rows of a whole-matrix quantization (and of the bias)."""
    a, b = shard_rows(packed.shape[0], world, rank)
    return (packed[a:b].contiguous(), scales[a:b].contiguous(),
            None if zeros is None else zeros[a:b].contiguous(),
            None if bias is None else bias[a:b].contiguous())


def _library_matmul(x, packed, scales, K, group, zeros, bias, relu):
    from . import int4_matmul
    return int4_matmul(x, packed, scales, K, group, zeros=zeros, bias=bias, relu=relu)


class ShardedInt4Linear(torch.nn.Module):
    """y = act(x @ dequantize(W)^T + bias) with W's rows split over a group.

    Built from this rank's shard (see shard_quantized).  `matmul` computes the
    local columns (default: the library's int4_matmul); the gather is one
    torch.distributed all_gather of equal-sized, zero-padded column blocks.
    """

    def __init__(self, packed, scales, zeros, bias, *, in_features: int, out_features: int,
                 group: int, relu: bool = False, process_group=None,
                 matmul: Callable | None = None):
        super().__init__()
        self.pg = process_group
        self.world = dist.get_world_size(process_group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(process_group) if dist.is_initialized() else 0
        self.in_features, self.out_features = int(in_features), int(out_features)
        self.group, self.relu = int(group), bool(relu)
        self.start, self.stop = shard_rows(self.out_features, self.world, self.rank)
        if packed.shape[0] != self.stop - self.start:
            raise ValueError("the shard's rows do not match shard_rows for this rank")
        self.packed, self.scales, self.zeros, self.bias = packed, scales, zeros, bias
        self.matmul = matmul if matmul is not None else _library_matmul
        self.max_rows = shard_rows(self.out_features, self.world, 0)[1]

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        lead = x.shape[:-1]
        x2 = x.reshape(-1, self.in_features)
        M = x2.shape[0]
        local = self.matmul(x2, self.packed, self.scales, self.in_features, self.group,
                            self.zeros, self.bias, self.relu)                  # [M, rows]
        if self.world == 1:
            return local.reshape(*lead, self.out_features)
        block = torch.zeros((M, self.max_rows), dtype=local.dtype, device=local.device)
        block[:, :local.shape[1]] = local
        blocks = [torch.empty_like(block) for _ in range(self.world)]
        dist.all_gather(blocks, block.contiguous(), group=self.pg)
        cols = []
        for p in range(self.world):
            a, b = shard_rows(self.out_features, self.world, p)
            cols.append(blocks[p][:, :b - a])
        return torch.cat(cols, dim=1).reshape(*lead, self.out_features)
