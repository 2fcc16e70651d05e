"""Column-parallel LLM.int8() linear layer: one process per GPU, each owning a
block of the weight's output columns.

The method has no exchange step when W is split by columns ("LLM.int8():
8-bit Matrix Multiplication for Transformers at Scale", Appendix D runs a
175B-size model over several GPUs this way). Every rank holds the whole
activation X and finds the same outlier columns, row scales and row codes
from it; each column's scale and int8 codes depend on that column alone, and
each output column on X and that column alone. So a rank that prepares
columns [col0, col0 + width) of W (llmint8_prepare_weight_cols, straight from
the full fp16 W, no copy) and runs llmint8_matmul on them produces exactly
that block of the layer's output, bit for bit, with no communication. A
contiguous output, when the caller wants one, is an all-gather of the blocks
over NCCL (torch.distributed) after the layer.

Every step of the layer runs in the CUDA library; this module only chooses
column blocks and moves the finished blocks.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch

from . import binding

COLUMN_ALIGN = 16  # columns per block are a multiple of this (the ABI's rule)


def shard_width(o: int, world: int, align: int = COLUMN_ALIGN) -> int:
    """Columns per rank: o / world rounded up to a multiple of `align` (the
    last rank's block may be narrower, or empty)."""
    if o <= 0 or world <= 0:
        raise ValueError("o and world must be positive")
    per = -(-o // world)
    return -(-per // align) * align


def shard_columns(o: int, world: int, rank: int,
                  align: int = COLUMN_ALIGN) -> Tuple[int, int]:
    """(col0, width) of rank's block of the o output columns."""
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside world {world}")
    per = shard_width(o, world, align)
    col0 = min(o, rank * per)
    return col0, max(0, min(o, col0 + per) - col0)


def gather_columns(block: torch.Tensor, o: int, world: int, group=None) -> torch.Tensor:
    """All-gather every rank's output block [s, width] into the layer's
    contiguous output [s, o] (on every rank). Blocks are padded to the common
    width for the collective and the padding is dropped."""
    import torch.distributed as dist

    s = block.shape[0]
    per = shard_width(o, world)
    if block.shape[1] < per:
        padded = block.new_zeros((s, per))
        padded[:, :block.shape[1]] = block
        block = padded
    parts = [torch.empty_like(block) for _ in range(world)]
    dist.all_gather(parts, block.contiguous(), group=group)
    return torch.cat(parts, dim=1)[:, :o].contiguous()


class ColumnParallelLinear:
    """This rank's block of an LLM.int8() layer.

    W is the full fp16 weight [h, o] on this rank's GPU (only the rank's
    columns are read); rank and world default to torch.distributed's."""

    def __init__(self, W: torch.Tensor, world: Optional[int] = None,
                 rank: Optional[int] = None, group=None, max_outliers: int = 0):
        if world is None or rank is None:
            import torch.distributed as dist
            world = dist.get_world_size(group) if world is None else world
            rank = dist.get_rank(group) if rank is None else rank
        self.h, self.o = W.shape
        self.world, self.rank, self.group = world, rank, group
        self.col0, self.width = shard_columns(self.o, world, rank)
        self.max_outliers = max_outliers
        self.pw = (binding.llmint8_prepare_weight_cols(W, self.col0, self.width)
                   if self.width > 0 else None)
        self._ws = None

    def workspace(self, s: int, device) -> binding.Workspace:
        if self._ws is None or self._ws.s < s:
            self._ws = binding.Workspace(s, self.h, self.width, device=device,
                                         max_outliers=self.max_outliers)
        return self._ws

    def __call__(self, X: torch.Tensor, alpha: float = 6.0,
                 gather: bool = False) -> torch.Tensor:
        """This rank's output block [s, width], or with gather the whole
        output [s, o] (an NCCL all-gather after the layer)."""
        s = X.shape[0]
        if self.width == 0:
            block = torch.empty((s, 0), dtype=torch.float16, device=X.device)
        else:
            block = binding.llmint8_matmul(X, self.pw, alpha,
                                           workspace=self.workspace(s, X.device))
        return gather_columns(block, self.o, self.world, self.group) if gather else block
