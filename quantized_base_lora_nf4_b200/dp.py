"""Data-parallel plumbing for the adapter training step (host side; torch.distributed).

The frozen quantised weight is replicated on every rank and never changes, so the only exchange a
data-parallel step needs is the adapter gradients.  Each rank's dA and dB are sums over its own
tokens (the layer's backward sums over tokens and applies no 1/M), so the full-batch gradient is the
plain SUM over ranks ("Background: how LoRA works": only A and B are trained).  The gradients travel
in flattened buckets, one collective per bucket: one bucket for a single layer or block, and for a
stack of layers buckets of about 32 MB whose exchange overlaps the backward of the later layers.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence, Tuple

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

    def start(self, group: Optional[dist.ProcessGroup] = None, stream=None):
        """Copy the gradients in and start the SUM all-reduce without waiting for it (None when there
        is nothing to exchange).  The copies and, with NCCL, the collective are ordered after the work
        already issued on `stream`: the CUDA stream the gradients were computed on (the library's calls
        take an explicit stream), torch's current stream when None.  They are issued on that stream, so
        the exchange never reads gradients the backward has not finished writing and does not hold up
        the other streams."""
        if not dist.is_initialized() or dist.get_world_size(group) == 1:
            return None
        if stream is not None and self.flat.is_cuda:
            with torch.cuda.stream(stream):
                return self._start(group)
        return self._start(group)

    def _start(self, group):
        off = 0
        for g, n in zip(self.grads, self.sizes):
            self.flat[off:off + n].copy_(g.reshape(-1))
            off += n
        return dist.all_reduce(self.flat, op=dist.ReduceOp.SUM, group=group, async_op=True)

    def wait(self, work) -> None:
        """Order the current stream after the all-reduce started by `start` and copy the sums out."""
        if work is None:
            return
        work.wait()
        off = 0
        for g, n in zip(self.grads, self.sizes):
            g.view(-1).copy_(self.flat[off:off + n])
            off += n

    def allreduce(self, group: Optional[dist.ProcessGroup] = None) -> None:
        self.wait(self.start(group))


class OverlappedBuckets:
    """The adapter gradients of a step grouped, in the order their layers finish the backward, into
    buckets of about `cap_bytes`.  A bucket's all-reduce starts as soon as its last layer is done
    (`layer_done`), so the exchange overlaps the backward of the layers after it; `finish` waits for
    all of them.  Every rank builds the same buckets and starts them in the same order."""

    def __init__(self, grads_per_layer: Sequence[Sequence[torch.Tensor]], cap_bytes: int = 32 << 20):
        if not grads_per_layer:
            raise ValueError("no layers")
        self.buckets: List[GradBucket] = []
        self.start_after: Dict[int, int] = {}  # layer index -> bucket started after that layer
        cur: List[torch.Tensor] = []
        cur_bytes = 0
        last = len(grads_per_layer) - 1
        for i, gs in enumerate(grads_per_layer):
            cur.extend(gs)
            cur_bytes += sum(g.numel() * g.element_size() for g in gs)
            if cur and (cur_bytes >= cap_bytes or i == last):
                self.start_after[i] = len(self.buckets)
                self.buckets.append(GradBucket(cur))
                cur, cur_bytes = [], 0
        self.pending: List[Tuple[int, object]] = []

    def layer_done(self, i: int, group: Optional[dist.ProcessGroup] = None, stream=None) -> None:
        """Layer i's backward has been issued (on `stream`, default torch's current stream)."""
        b = self.start_after.get(i)
        if b is not None:
            self.pending.append((b, self.buckets[b].start(group, stream)))

    def finish(self) -> None:
        for b, work in self.pending:
            self.buckets[b].wait(work)
        self.pending = []


def allreduce_adapter_grads(grads: Sequence[torch.Tensor], group: Optional[dist.ProcessGroup] = None) -> None:
    """SUM-reduce the adapter gradients of one step across ranks, in place (one collective)."""
    GradBucket(grads).allreduce(group)
