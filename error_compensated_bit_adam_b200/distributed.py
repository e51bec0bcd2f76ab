"""1-bit Adam over G processes, one per GPU, through the split step.

The compressed collective of the review page "1-bit Adam: Communication
Efficient Large-Scale Training with Adam's Convergence Speed" ("Proposed
method", 4) has a worker stage (every worker compresses its momentum and
sends its words and scale onward) and a server stage (the compressed
momenta are averaged, compressed again and returned to every worker).
Here process r of G computes the worker stage of workers
[r W/G, (r+1) W/G) with ob_worker_stage, the worker rows (sign words and
scales) are all-gathered, and every process then runs the server stage of
every chunk and the update with ob_finish_step.  Given the same rows, every
process computes the same server words, so nothing is sent back, and every
process ends the step with the same parameters, bit for bit equal to one
ob_compressed_step over all W workers.

Against the pages' exchange (each server receives only its chunk of every
worker's words and returns its chunk to every worker) this sends each
process every worker's whole row and repeats the server stage on every
process: one collective over the library's own layout, and no kernel
beyond the single-GPU step's.

LocalRanks runs the same split step for G ranks inside one process on one
GPU, each rank a context of its own, with the all-gather done by device
copies: the single-GPU form of the path, used to check it against one
context and to time each rank's share of the work.
"""
from __future__ import annotations

from typing import List, Optional, Sequence

import torch

from . import _binding as B
from .optimizer import OneBitAdam


def _view(workspace: torch.Tensor, ptr: int, nbytes: int, dtype: torch.dtype) -> torch.Tensor:
    """The bytes [ptr, ptr + nbytes) of the workspace as a flat tensor."""
    off = ptr - workspace.data_ptr()
    assert 0 <= off and off + nbytes <= workspace.numel()
    return workspace[off:off + nbytes].view(dtype)


class TorchExchange:
    """The split step's exchange over a torch.distributed group (NCCL for
    CUDA tensors, gloo for CPU tensors).  The collective runs on the current
    stream; every rank calls it in the same order."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def gather_rows(self, rows: torch.Tensor, begin: int, count: int) -> None:
        """rows: [R, k], rank q's block at rows [q count, (q+1) count); this
        rank's block (begin = rank * count) is gathered in place into all."""
        assert rows.shape[0] == count * self.world and begin == self.rank * count
        flat = rows.view(-1)
        mine = rows[begin:begin + count].view(-1)
        self.dist.all_gather_into_tensor(flat, mine, group=self.group)


class DistributedOneBitAdam:
    """One process's part of a data-parallel 1-bit Adam run.

    numel, W, hyperparameters: as for OneBitAdam (W % world == 0).  Each
    process keeps a context over the whole tensor list with all W workers
    (parameters, momentum and variance are the same everywhere).  The phase
    methods below are the split step; ``step`` runs them with ``exchange``
    (a TorchExchange by default) between the two library calls."""

    def __init__(self, numel: Sequence[int], W: int, *, rank: int, world: int, exchange=None,
                 device=None, stream: Optional[torch.cuda.Stream] = None, **hyper):
        if world < 1 or W % world != 0 or not 0 <= rank < world:
            raise ValueError(f"W = {W} workers cannot be split over {world} processes")
        self.rank, self.world = int(rank), int(world)
        self.W = int(W)
        self.w_local = self.W // self.world
        self.w_begin = self.rank * self.w_local
        self.exchange_impl = exchange
        self.opt = OneBitAdam(numel, W, device=device, stream=stream, **hyper)
        ctx, ws = self.opt.ctx, self.opt.workspace
        bits, bits_row, scales, scales_row = B.ob_worker_exchange_buffers(ctx)
        self.worker_bits = _view(ws, bits, self.W * bits_row, torch.int32).view(self.W, -1)
        self.worker_scales = _view(ws, scales, self.W * scales_row, torch.float32).view(self.W, -1)

    @property
    def params(self) -> torch.Tensor:
        return self.opt.params

    def layout(self):
        return self.opt.layout()

    # --------------------------------------------------------- warmup
    def warmup_step(self, all_grads: torch.Tensor) -> None:
        """Full-precision Adam on the average of all W workers' gradients,
        [W, n_padded] (the warmup adds them in worker order, so every
        process needs all of them)."""
        self.opt.warmup_step(all_grads)

    def freeze(self) -> None:
        self.opt.freeze()

    # ------------------------------------------------------ split step
    def worker_stage(self, local_grads: Sequence[torch.Tensor]) -> None:
        """This process's workers: local_grads[i] is worker w_begin + i's
        gradient (contiguous float32 CUDA, n_padded elements)."""
        if len(local_grads) != self.w_local:
            raise ValueError(f"expected {self.w_local} local gradients")
        ptrs = [0] * self.W
        for i, g in enumerate(local_grads):
            if (g.dtype != torch.float32 or not g.is_cuda or not g.is_contiguous()
                    or g.numel() != self.opt.n_padded):
                raise ValueError("each gradient must be a contiguous float32 CUDA vector of "
                                 f"{self.opt.n_padded} elements")
            ptrs[self.w_begin + i] = g.data_ptr()
        B.ob_worker_stage(self.opt.ctx, ptrs, self.w_begin, self.w_local)

    def finish_step(self) -> None:
        B.ob_finish_step(self.opt.ctx)

    def exchange(self, ex) -> None:
        ex.gather_rows(self.worker_bits, self.w_begin, self.w_local)
        ex.gather_rows(self.worker_scales, self.w_begin, self.w_local)

    def step(self, local_grads: Sequence[torch.Tensor]) -> None:
        ex = self.exchange_impl if self.exchange_impl is not None else TorchExchange()
        with torch.cuda.stream(self.opt.stream):
            self.worker_stage(local_grads)
            self.exchange(ex)
            self.finish_step()

    def exchange_bytes(self) -> int:
        """Bytes the all-gather brings into this process per step."""
        return (self.W - self.w_local) * (self.worker_bits.shape[1] + self.worker_scales.shape[1]) * 4

    def read(self, kind: int, index: int = 0):
        return self.opt.read(kind, index)

    def close(self) -> None:
        self.opt.close()


class LocalRanks:
    """G ranks of the split step in one process on one GPU, stepped in
    lockstep; the all-gather is device copies.  No kernel of one rank waits
    for another's: the ranks' launches are queued one after another on the
    same stream."""

    def __init__(self, numel: Sequence[int], W: int, G: int, device=None, **hyper):
        self.G, self.W = int(G), int(W)
        stream = torch.cuda.current_stream(device)
        self.ranks: List[DistributedOneBitAdam] = [
            DistributedOneBitAdam(numel, W, rank=r, world=G, device=device, stream=stream, **hyper)
            for r in range(G)]
        self.w_local = self.ranks[0].w_local

    def warmup_step(self, all_grads: torch.Tensor) -> None:
        for r in self.ranks:
            r.warmup_step(all_grads)

    def freeze(self) -> None:
        for r in self.ranks:
            r.freeze()

    def _gather_rows(self, attr: str) -> None:
        for dst in self.ranks:
            for src in self.ranks:
                if src is not dst:
                    rows = slice(src.w_begin, src.w_begin + src.w_local)
                    getattr(dst, attr)[rows].copy_(getattr(src, attr)[rows])

    def step(self, all_grads: torch.Tensor) -> None:
        """all_grads: [W, n_padded]; rank r gets its workers' rows."""
        for r in self.ranks:
            r.worker_stage([all_grads[r.w_begin + i] for i in range(r.w_local)])
        self._gather_rows("worker_bits")
        self._gather_rows("worker_scales")
        for r in self.ranks:
            r.finish_step()

    def close(self) -> None:
        for r in self.ranks:
            r.close()
