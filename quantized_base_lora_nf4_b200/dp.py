"""Data-parallel plumbing for the adapter training step (host side; torch.distributed).

The frozen quantised weight is replicated on every rank and never changes, so the only exchange a
data-parallel step needs is the adapter gradients.  Each rank's dA and dB are sums over its own
tokens (the layer's backward sums over tokens and applies no 1/M), so the full-batch gradient is the
plain SUM over ranks ("Background: how LoRA works": only A and B are trained).  The gradients of all
adapters of a step travel in one flattened buffer, so a step issues one collective whatever the
number of adapters.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist


def shard_rows(total: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous, balanced token range [start, stop) of `rank` among `world` ranks."""
    if world < 1 or not 0 <= rank < world or total < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


class GradBucket:
    """One flat buffer holding a fixed list of gradient tensors (same dtype and device), reduced with
    one all-reduce per step.  The tensors keep their own storage; the bucket copies in and out."""

    def __init__(self, grads: Sequence[torch.Tensor]):
        if not grads:
            raise ValueError("empty bucket")
        dt, dev = grads[0].dtype, grads[0].device
        if any(g.dtype != dt or g.device != dev for g in grads):
            raise ValueError("a bucket holds one dtype on one device")
        self.grads: List[torch.Tensor] = list(grads)
        self.sizes = [g.numel() for g in self.grads]
        self.flat = torch.empty(sum(self.sizes), dtype=dt, device=dev)

    def allreduce(self, group: Optional[dist.ProcessGroup] = None) -> None:
        if not dist.is_initialized() or dist.get_world_size(group) == 1:
            return
        off = 0
        for g, n in zip(self.grads, self.sizes):
            self.flat[off:off + n].copy_(g.reshape(-1))
            off += n
        dist.all_reduce(self.flat, op=dist.ReduceOp.SUM, group=group)
        off = 0
        for g, n in zip(self.grads, self.sizes):
            g.view(-1).copy_(self.flat[off:off + n])
            off += n


def allreduce_adapter_grads(grads: Sequence[torch.Tensor], group: Optional[dist.ProcessGroup] = None) -> None:
    """SUM-reduce the adapter gradients of one step across ranks, in place (one collective)."""
    GradBucket(grads).allreduce(group)
