"""Bucketed compressed steps that overlap the backward pass.

The compression-phase step of 1-bit Adam works tensor by tensor (scales,
sign packing and server chunks are all per tensor), so a parameter list can
be cut into buckets, each stepped by its own context on its own CUDA
stream as soon as that bucket's gradients exist -- while the backward pass
is still computing the gradients of earlier layers.  The results are
bit-identical to one context over the whole list.  This is the overlap
behind the end-to-end throughput the review page "1-bit Adam:
Communication Efficient Large-Scale Training with Adam's Convergence
Speed" reports ("Key results"): the optimizer step, HBM-bound, runs beside
the tensor-core-bound backward GEMMs.
"""
from __future__ import annotations

from typing import List, Optional, Sequence

import torch

from .optimizer import Grads, OneBitAdam


def split_buckets(numel: Sequence[int], bucket_elems: int) -> List[List[int]]:
    """Consecutive tensors grouped into buckets of about bucket_elems
    elements (a tensor larger than that is a bucket of its own).  Returns
    the tensor indices of each bucket, in order."""
    buckets, cur, size = [], [], 0
    for t, n in enumerate(numel):
        if cur and size + n > bucket_elems:
            buckets.append(cur)
            cur, size = [], 0
        cur.append(t)
        size += n
    if cur:
        buckets.append(cur)
    return buckets


class BucketedOneBitAdam:
    """One OneBitAdam context per bucket, each on its own CUDA stream.

    buckets: tensor indices per bucket (see split_buckets).  Each bucket's
    gradients are a [W, n_padded(bucket)] tensor in that bucket's padded
    layout (``layout(b)``).  ``step(b, grads, ready)`` queues bucket b's
    compressed step on its stream after the CUDA event `ready` (recorded on
    the producer's stream when the gradients are complete); ``wait()``
    makes the current stream wait for every bucket.  graph=True replays
    each bucket's step as one CUDA graph; priority < 0 gives the bucket
    streams a higher scheduling priority than default streams.  The caller
    must not overwrite a bucket's gradients before its step has run (wait()
    or an event of the bucket's stream).
    """

    def __init__(self, numel: Sequence[int], W: int, buckets: Sequence[Sequence[int]], *,
                 graph: bool = True, device=None, priority: int = 0, **hyper):
        self.numel = [int(n) for n in numel]
        self.buckets = [list(b) for b in buckets]
        assert sorted(t for b in self.buckets for t in b) == list(range(len(self.numel)))
        self.W = int(W)
        self.device = torch.device(device if device is not None else "cuda")
        self.streams = [torch.cuda.Stream(device=self.device, priority=priority)
                        for _ in self.buckets]
        self.opts = [OneBitAdam([self.numel[t] for t in b], W, device=self.device, stream=s, **hyper)
                     for b, s in zip(self.buckets, self.streams)]
        for o in self.opts:
            o.graph(graph)

    def layout(self, b: int):
        return self.opts[b].layout()

    def params(self, b: int) -> torch.Tensor:
        return self.opts[b].params

    def _after(self, b: int, ready: Optional[torch.cuda.Event]) -> None:
        if ready is not None:
            self.streams[b].wait_event(ready)
        else:
            self.streams[b].wait_stream(torch.cuda.current_stream(self.device))

    def warmup_step(self, b: int, grads: Grads, ready: Optional[torch.cuda.Event] = None) -> None:
        self._after(b, ready)
        self.opts[b].warmup_step(grads)

    def freeze(self) -> None:
        for o in self.opts:
            o.freeze()

    def step(self, b: int, grads: Grads, ready: Optional[torch.cuda.Event] = None) -> None:
        self._after(b, ready)
        self.opts[b].step(grads)

    def wait(self) -> None:
        cur = torch.cuda.current_stream(self.device)
        for s in self.streams:
            cur.wait_stream(s)

    def close(self) -> None:
        for o in self.opts:
            o.close()
