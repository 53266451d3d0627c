"""Data-parallel gradient exchange of block-circulant layers.

Tokens are sharded over ranks; y and grad_x stay local, and the only exchange is the
sum over ranks of each layer's grad_c (a sum over tokens, so the per-rank sums add
up). All grad_c buffers of a step are exchanged in one bucket: copied into one flat
buffer, all-reduced once (NCCL over NVLink between GPUs, gloo on CPU), copied back.
Because rdIFFT is linear it does not matter whether the packed cross-spectrum or the
spatial grad_c is summed; the spatial grad_c that circ_bwd returns is summed here.
"""
from __future__ import annotations

from typing import Sequence

import torch
import torch.distributed as dist


class GradCBucket:
    """A flat buffer holding views of every grad_c of a step, all-reduced at once."""

    def __init__(self, shapes: Sequence[torch.Size], device, dtype=torch.float32):
        self.numels = [int(torch.Size(s).numel()) for s in shapes]
        self.flat = torch.zeros(sum(self.numels), device=device, dtype=dtype)
        self.views = []
        off = 0
        for s, n in zip(shapes, self.numels):
            self.views.append(self.flat[off:off + n].view(s))
            off += n

    def allreduce(self, group=None, world_size: int | None = None, average: bool = False):
        """Sums (or averages) the bucket over the ranks of `group` in place."""
        if world_size is None:
            world_size = dist.get_world_size(group) if dist.is_initialized() else 1
        if world_size > 1:
            dist.all_reduce(self.flat, op=dist.ReduceOp.SUM, group=group)
        if average and world_size > 1:
            self.flat.div_(world_size)
        return self.views


def shard_tokens(total_tokens: int, rank: int, world_size: int) -> slice:
    """Contiguous token range of a rank (the first ranks take one more when uneven)."""
    base, extra = divmod(total_tokens, world_size)
    start = rank * base + min(rank, extra)
    return slice(start, start + base + (1 if rank < extra else 0))
