"""Data parallelism for the QLoRA linear: token shards and the exchange of the
adapter gradients.

Every rank holds a whole replica of the encoded base weight and of the
adapter (A, B) and runs the layer on its own tokens: data-parallel training
keeps one full quantised base per process ("第 04 篇：QLoRA 原理" §10.4).  Y and
dX stay on the rank that computed them.  The adapter gradients

    dA = s (dY B)^T X,    dB = s dY^T (X A^T)

are sums over tokens (§2.4, §6.4), so the gradient of the whole batch is the
SUM over ranks of the gradients of the shards: the one exchange step of the
path, an all-reduce.  The base weight has no gradient and is never exchanged.

`torch.distributed` carries the collective (NCCL over NVLink on GPUs, gloo on
CPU); this module only decides the shards and packs the gradients so that one
call per step moves them all.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist


def token_shard(M: int, world: int, rank: int) -> Tuple[int, int]:
    """[begin, end) of rank's tokens: contiguous, sizes differ by at most one,
    the first M % world ranks take one more.  A rank may get none (M < world):
    its backward then contributes zero gradients (the layer's empty batch)."""
    if world < 1 or not 0 <= rank < world or M < 0:
        raise ValueError("need world >= 1, 0 <= rank < world, M >= 0")
    per, extra = divmod(M, world)
    begin = rank * per + min(rank, extra)
    return begin, begin + per + (1 if rank < extra else 0)


class LoraGradExchange:
    """SUM all-reduce of a fixed list of adapter gradients, in place.

    The tensors (bf16 or fp32, any shapes, all on one device) are packed into
    one fp32 buffer, reduced with a single collective and written back: the
    cross-rank sum is formed in fp32 and each bf16 gradient is rounded once,
    to nearest even, at the end.  `average=True` divides by the group size
    (the mean over ranks instead of the sum)."""

    def __init__(self, grads: Sequence[torch.Tensor], group: Optional[dist.ProcessGroup] = None):
        if not grads:
            raise ValueError("no gradients to exchange")
        dev = grads[0].device
        for g in grads:
            if g.device != dev or g.dtype not in (torch.bfloat16, torch.float32) or not g.is_contiguous():
                raise ValueError("gradients must be contiguous bf16/fp32 tensors on one device")
        self.grads: List[torch.Tensor] = list(grads)
        self.group = group
        self.offsets = []
        n = 0
        for g in self.grads:
            self.offsets.append(n)
            n += g.numel()
        self.flat = torch.empty(n, dtype=torch.float32, device=dev)

    @property
    def numel(self) -> int:
        return self.flat.numel()

    def __call__(self, average: bool = False) -> None:
        for g, off in zip(self.grads, self.offsets):
            self.flat[off:off + g.numel()].copy_(g.reshape(-1))
        dist.all_reduce(self.flat, op=dist.ReduceOp.SUM, group=self.group)
        if average:
            self.flat.div_(dist.get_world_size(self.group))
        for g, off in zip(self.grads, self.offsets):
            g.reshape(-1).copy_(self.flat[off:off + g.numel()])


class OverlappedGradExchange:
    """The exchange split per module and overlapped with the rest of the
    backward ("第 04 篇：QLoRA 原理" §10.4: one full quantised base per
    data-parallel process; only the adapter gradients cross ranks).

    `buckets[i]` lists module i's gradients (its dA and dB).  As soon as the
    backward of module i has produced them on the current stream,
    ``launch(i)`` records an event there and, on a side stream that waits for
    that event, packs them, SUM-all-reduces them and writes them back, while
    the current stream goes on with the next module.  ``finish()`` makes the
    current stream wait for every exchange launched so far: call it before
    anything reads or overwrites the gradients again (the optimizer step, the
    next step's backward).  On CPU tensors (gloo) there are no streams and
    ``launch`` exchanges at once.  Each bucket is reduced in fp32 and each
    bf16 gradient rounded once, as in LoraGradExchange."""

    def __init__(self, buckets: Sequence[Sequence[torch.Tensor]], group: Optional[dist.ProcessGroup] = None,
                 stream: Optional["torch.cuda.Stream"] = None):
        if not buckets:
            raise ValueError("no gradient buckets")
        self.buckets = [LoraGradExchange(b, group) for b in buckets]
        dev = self.buckets[0].flat.device
        if any(b.flat.device != dev for b in self.buckets):
            raise ValueError("all buckets must be on one device")
        self.cuda = dev.type == "cuda"
        self.stream = (stream if stream is not None else torch.cuda.Stream(device=dev)) if self.cuda else None
        self.launched = 0

    def launch(self, i: int, average: bool = False) -> None:
        bucket = self.buckets[i]
        if not self.cuda:
            bucket(average)
            return
        ready = torch.cuda.Event()
        ready.record(torch.cuda.current_stream(self.stream.device))
        with torch.cuda.stream(self.stream):
            self.stream.wait_event(ready)  # module i's gradients are complete
            bucket(average)
        self.launched += 1

    def finish(self) -> None:
        if self.cuda and self.launched:
            torch.cuda.current_stream(self.stream.device).wait_stream(self.stream)
            self.launched = 0


def max_over_ranks(value: float, device: torch.device, group: Optional[dist.ProcessGroup] = None) -> float:
    """The largest `value` of all ranks (a step time: the slowest rank sets
    the pace of a synchronous data-parallel step)."""
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
