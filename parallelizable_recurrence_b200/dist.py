"""Data-parallel plumbing for the SRU layer step: one process per GPU.

The SRU layer shards naturally over the batch: every (batch row, channel)
stream is independent once U exists ("When Attention Meets Fast Recurrence",
background section on SRU), so the forward needs no exchange.  In a training
step the parameter gradients dW_cat, v and b are sums over the batch rows, so
ranks that each hold a shard of the rows sum those gradients with one
all-reduce -- the distributed data parallelism the page's experiments use.

This module holds only that plumbing (which rows a rank owns, and the packed
all-reduce); the arithmetic of the layer stays in the CUDA library.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import torch
import torch.distributed as dist


def batch_shard(total_rows: int, world: int, rank: int) -> Tuple[int, int]:
    """[start, stop) of the batch rows owned by `rank`: contiguous, sizes differ by at most one."""
    if world < 1 or not (0 <= rank < world) or total_rows < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(total_rows, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


class GradReducer:
    """Sums a fixed set of gradient tensors over all ranks with ONE all-reduce.

    The tensors are packed into one flat buffer (allocated once), reduced in
    place with SUM, and unpacked back into the original tensors.  Every rank
    must construct it with tensors of the same shapes, in the same order, and
    call it the same number of times (collectives are matched by order).
    """

    def __init__(self, tensors: Sequence[torch.Tensor]):
        if not tensors:
            raise ValueError("no tensors to reduce")
        dev, dt = tensors[0].device, tensors[0].dtype
        for t in tensors:
            if t.device != dev or t.dtype != dt or not t.is_contiguous():
                raise ValueError("gradients must share device and dtype and be contiguous")
        self.tensors: List[torch.Tensor] = list(tensors)
        self.numels = [t.numel() for t in tensors]
        self.flat = torch.empty(sum(self.numels), device=dev, dtype=dt)

    def __call__(self, group=None) -> None:
        off = 0
        for t, n in zip(self.tensors, self.numels):
            self.flat[off:off + n].copy_(t.view(-1))
            off += n
        dist.all_reduce(self.flat, op=dist.ReduceOp.SUM, group=group)
        off = 0
        for t, n in zip(self.tensors, self.numels):
            t.view(-1).copy_(self.flat[off:off + n])
            off += n
