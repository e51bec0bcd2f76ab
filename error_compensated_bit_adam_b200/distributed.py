"""1-bit Adam over G processes, one per GPU, through the split step.

The compressed collective of the review page "1-bit Adam: Communication
Efficient Large-Scale Training with Adam's Convergence Speed" ("Proposed
method", 4) has a worker stage (every worker compresses its momentum and
sends server j the part of its words that chunk j covers) and a server
stage (server j averages its chunk, compresses it again and sends the
result to every worker).  Here process r of G computes workers
[r W/G, (r+1) W/G) and serves one contiguous range of the server chunks,
whose words are one contiguous range [wb_r, we_r) of the padded layout
(ob_server_shard_range).  Between the library's three calls
(ob_worker_stage, ob_server_stage, ob_apply_update) the process exchanges

  * chunks of the worker words: process r sends words [wb_q, we_q) of each
    of its workers' rows to process q and receives words [wb_r, we_r) of
    every other worker's row (grouped point-to-point sends and receives:
    about (W - W/G) n / (8 G) bytes in per process), plus an all-gather of
    the worker scales (W x T floats);
  * the server results: process r sends its words [wb_r, we_r) and its
    chunks' scales to every other process and receives theirs (about n/8
    bytes in per process).

With peer_words (ob_set_peer_words) the two word exchanges move into the
kernels instead: the worker stage stores each chunk's words straight into
the serving process's rows, and the update reads each chunk's server words
from the serving process (copying them locally); only the worker scales
and the server scales are still exchanged, and those exchanges also order
the stages across processes; a process's worker rows, its own workers'
included, then hold only the words of the chunks it serves.  The other
processes' buffers are mapped into each process with CUDA IPC.

Every process ends the step with the same parameters, bit for bit equal to
one ob_compressed_step over all W workers.  A process's rows of the other
workers hold only the words of the chunks it serves (the rest is stale),
and its server error only the chunks it serves.

LocalRanks runs the same split step for G ranks inside one process on one
GPU, each rank a context of its own, with the exchanges done by device
copies of the same ranges: the single-GPU form of the path, used to check
it against one context and to time each rank's share of the work.
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
    """The split step's exchanges over a torch.distributed group (NCCL for
    CUDA tensors, gloo for CPU tensors).  They run on the current stream;
    every rank calls them in the same order with the same ranges."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def _peer(self, q: int) -> int:
        return q if self.group is None else self.dist.get_global_rank(self.group, q)

    def _run(self, ops) -> None:
        if ops:
            for req in self.dist.batch_isend_irecv(ops):
                req.wait()

    def gather_rows(self, rows: torch.Tensor, begin: int, count: int) -> None:
        """rows: [R, k], rank q's block at rows [q count, (q+1) count); this
        rank's block (begin = rank * count) is gathered in place into all."""
        assert rows.shape[0] == count * self.world and begin == self.rank * count
        flat = rows.view(-1)
        mine = rows[begin:begin + count].view(-1)
        self.dist.all_gather_into_tensor(flat, mine, group=self.group)

    def send_worker_chunks(self, rows: torch.Tensor, count: int, ranges) -> None:
        """Worker stage: rows [W, words], rank q's workers at rows
        [q count, (q+1) count), rank q serving columns ranges[q] = (a, b).
        Afterwards every rank holds columns ranges[rank] of every row."""
        P2P = self.dist.P2POp
        r, ops = self.rank, []
        for q in range(self.world):
            if q == r:
                continue
            a, b = ranges[q]
            if b > a:        # my workers' words of q's chunks, to q
                ops += [P2P(self.dist.isend, rows[w, a:b], self._peer(q), self.group)
                        for w in range(r * count, (r + 1) * count)]
            a, b = ranges[r]
            if b > a:        # q's workers' words of my chunks, from q
                ops += [P2P(self.dist.irecv, rows[w, a:b], self._peer(q), self.group)
                        for w in range(q * count, (q + 1) * count)]
        self._run(ops)

    def gather_ranges(self, buf: torch.Tensor, ranges) -> None:
        """Server stage: buf is 1-D, rank q holding the entries ranges[q] =
        (a, b).  Afterwards every rank holds all of them."""
        P2P = self.dist.P2POp
        r, ops = self.rank, []
        a_r, b_r = ranges[r]
        for q in range(self.world):
            if q == r:
                continue
            if b_r > a_r:
                ops.append(P2P(self.dist.isend, buf[a_r:b_r], self._peer(q), self.group))
            a, b = ranges[q]
            if b > a:
                ops.append(P2P(self.dist.irecv, buf[a:b], self._peer(q), self.group))
        self._run(ops)

    def sum_(self, buf: torch.Tensor) -> None:
        self.dist.all_reduce(buf, op=self.dist.ReduceOp.SUM, group=self.group)


def exchange_plan(numel: Sequence[int], W: int, world: int):
    """Per rank (chunk_begin, chunk_end) and (word_begin, word_end) of the
    server shard it serves (ob_server_shard_range)."""
    shards = [B.ob_server_shard_range(numel, W, world, q) for q in range(world)]
    return [(s[0], s[1]) for s in shards], [(s[2], s[3]) for s in shards]


class DistributedOneBitAdam:
    """One process's part of a data-parallel 1-bit Adam run.

    numel, W, hyperparameters: as for OneBitAdam (W % world == 0).  Each
    process keeps a context over the whole tensor list with all W workers
    (parameters, momentum and variance are the same everywhere).  The phase
    methods below are the split step; ``step`` runs them with ``exchange``
    (a TorchExchange by default) between the library calls."""

    def __init__(self, numel: Sequence[int], W: int, *, rank: int, world: int, exchange=None,
                 device=None, stream: Optional[torch.cuda.Stream] = None, peer_words: bool = False,
                 **hyper):
        if world < 1 or W % world != 0 or not 0 <= rank < world:
            raise ValueError(f"W = {W} workers cannot be split over {world} processes")
        self.rank, self.world = int(rank), int(world)
        self.W = int(W)
        self.w_local = self.W // self.world
        self.w_begin = self.rank * self.w_local
        self.exchange_impl = exchange
        self._zeros: Optional[torch.Tensor] = None
        self.opt = OneBitAdam(numel, W, device=device, stream=stream, **hyper)
        ctx, ws = self.opt.ctx, self.opt.workspace
        B.ob_set_server_shard(ctx, self.world, self.rank)
        # every rank's served chunks and their words, for the exchanges
        self.chunk_ranges, self.word_ranges = exchange_plan(numel, W, self.world)
        self.chunk_begin, self.chunk_end = self.chunk_ranges[self.rank]
        bits, bits_row, scales, scales_row = B.ob_worker_exchange_buffers(ctx)
        self.worker_bits = _view(ws, bits, self.W * bits_row, torch.int32).view(self.W, -1)
        self.worker_scales = _view(ws, scales, self.W * scales_row, torch.float32).view(self.W, -1)
        sbits, sbits_bytes, sp, sp_bytes = B.ob_server_exchange_buffers(ctx)
        self.server_bits = _view(ws, sbits, sbits_bytes, torch.int32)
        self.server_scales = _view(ws, sp, sp_bytes, torch.float32)
        self.peer_words = False
        self._peer_workspaces: List[torch.Tensor] = []
        if peer_words:
            self.connect_peers()

    def set_peer_words(self, worker_bits: Sequence[int], server_bits: Sequence[int]) -> None:
        """Fused word exchanges with the given per-shard buffer addresses
        (every process's worker_bits and server_bits, as this process
        addresses them)."""
        B.ob_set_peer_words(self.opt.ctx, list(worker_bits), list(server_bits))
        self.peer_words = True

    def connect_peers(self) -> None:
        """Map every process's workspace into this one with CUDA IPC (the
        handles travel over the default process group) and turn on the
        fused word exchanges.  Processes on one node whose GPUs reach each
        other's memory; not run on more than one GPU here."""
        import torch.distributed as dist
        from torch.multiprocessing.reductions import reduce_tensor
        ws = self.opt.workspace
        handles = [None] * self.world
        dist.all_gather_object(handles, reduce_tensor(ws) if self.world > 1 else None)
        peers = [ws if q == self.rank else h[0](*h[1]) for q, h in enumerate(handles)]
        self._peer_workspaces = peers                  # keeps the mappings alive
        bits_off = self.worker_bits.data_ptr() - ws.data_ptr()
        sbits_off = self.server_bits.data_ptr() - ws.data_ptr()
        self.set_peer_words([p.data_ptr() + bits_off for p in peers],
                            [p.data_ptr() + sbits_off for p in peers])

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

    def warmup_step_allreduce(self, local_grads: Sequence[torch.Tensor]) -> None:
        """Full-precision Adam on the average of all W workers' gradients
        with the sum taken by an all-reduce, as in ordinary data-parallel
        training: local_grads[i] (worker w_begin + i) is overwritten by the
        sum over processes of every process's i-th gradient, and the warmup
        kernel averages those W/G sums and W - W/G zero vectors (adding
        zeros is exact).  Equal to warmup_step up to the order of the
        additions inside the all-reduce."""
        if len(local_grads) != self.w_local:
            raise ValueError(f"expected {self.w_local} local gradients")
        with torch.cuda.stream(self.opt.stream):
            if self.world > 1:  # one process: the sums are its own gradients
                ex = self._exchange()
                for g in local_grads:
                    ex.sum_(g)
            self.warmup_from_sums(local_grads)

    def warmup_from_sums(self, sums: Sequence[torch.Tensor]) -> None:
        """The warmup step given the all-reduced sums of warmup_step_allreduce."""
        if self._zeros is None:
            self._zeros = torch.zeros(self.opt.n_padded, dtype=torch.float32, device=self.opt.device)
        rows = list(sums) + [self._zeros] * (self.W - len(sums))
        self.opt.warmup_step(rows)

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

    def server_stage(self) -> None:
        B.ob_server_stage(self.opt.ctx)

    def apply_update(self) -> None:
        B.ob_apply_update(self.opt.ctx)

    def serves(self, t: int, j: int) -> bool:
        """Whether this process serves chunk j of tensor t."""
        return self.chunk_begin <= t * self.W + j < self.chunk_end

    def _exchange(self):
        if self.exchange_impl is None:  # the default process group, made on first use
            self.exchange_impl = TorchExchange()
        return self.exchange_impl

    def exchange_worker_stage(self, ex) -> None:
        """The worker stage's exchange: each rank's chunks of every worker's
        words (unless the kernel stored them already), and all worker
        scales."""
        if not self.peer_words:
            ex.send_worker_chunks(self.worker_bits, self.w_local, self.word_ranges)
        ex.gather_rows(self.worker_scales, self.w_begin, self.w_local)

    def exchange_server_stage(self, ex) -> None:
        """The server stage's exchange: every rank's server words (unless the
        update reads them from their server) and chunk scales to every
        rank."""
        if not self.peer_words:
            ex.gather_ranges(self.server_bits, self.word_ranges)
        ex.gather_ranges(self.server_scales, self.chunk_ranges)

    def step(self, local_grads: Sequence[torch.Tensor]) -> None:
        ex = self._exchange() if self.world > 1 else None  # one process: nothing to exchange
        with torch.cuda.stream(self.opt.stream):
            self.worker_stage(local_grads)
            if ex is not None:
                self.exchange_worker_stage(ex)
            self.server_stage()
            if ex is not None:
                self.exchange_server_stage(ex)
            self.apply_update()

    def exchange_bytes(self) -> dict:
        """Bytes each exchange brings into this process per step (with
        peer_words the words move inside the kernels: stored by the other
        processes' worker stages, loaded by this process's update)."""
        others = self.W - self.w_local
        wb, we = self.word_ranges[self.rank]
        T = self.worker_scales.shape[1]
        theirs = [q for q in range(self.world) if q != self.rank]
        return {"worker_words": others * (we - wb) * 4,
                "worker_scales": others * T * 4,
                "server_words": sum(self.word_ranges[q][1] - self.word_ranges[q][0] for q in theirs) * 4,
                "server_scales": sum(self.chunk_ranges[q][1] - self.chunk_ranges[q][0]
                                     for q in theirs) * 4,
                "words_in_kernels": self.peer_words}

    def read(self, kind: int, index: int = 0):
        return self.opt.read(kind, index)

    def close(self) -> None:
        self.opt.close()


class LocalRanks:
    """G ranks of the split step in one process on one GPU, stepped in
    lockstep; the exchanges are device copies and sums.  No kernel of one
    rank waits for another's: the ranks' launches are queued one after
    another on the same stream."""

    def __init__(self, numel: Sequence[int], W: int, G: int, device=None, peer_words: bool = False,
                 **hyper):
        self.G, self.W = int(G), int(W)
        stream = torch.cuda.current_stream(device)
        self.ranks: List[DistributedOneBitAdam] = [
            DistributedOneBitAdam(numel, W, rank=r, world=G, device=device, stream=stream, **hyper)
            for r in range(G)]
        self.w_local = self.ranks[0].w_local
        self.peer_words = bool(peer_words)
        if self.peer_words:  # the "peers" are the other contexts' buffers on this GPU
            bits = [r.worker_bits.data_ptr() for r in self.ranks]
            sbits = [r.server_bits.data_ptr() for r in self.ranks]
            for r in self.ranks:
                r.set_peer_words(bits, sbits)

    def warmup_step(self, all_grads: torch.Tensor) -> None:
        for r in self.ranks:
            r.warmup_step(all_grads)

    def warmup_step_allreduce(self, all_grads: torch.Tensor) -> None:
        """warmup_step_allreduce of every rank, the all-reduce emulated by
        sums in rank order (all_grads is left unchanged)."""
        sums = []
        for i in range(self.w_local):
            t = all_grads[i].clone()
            for r in self.ranks[1:]:
                t += all_grads[r.w_begin + i]
            sums.append(t)
        for r in self.ranks:
            r.warmup_from_sums(sums)

    def freeze(self) -> None:
        for r in self.ranks:
            r.freeze()

    def _send_worker_chunks(self) -> None:
        """Rank dst receives, in every other rank's worker rows, the words
        of the chunks dst serves."""
        for dst in self.ranks:
            a, b = dst.word_ranges[dst.rank]
            if b <= a:
                continue
            for src in self.ranks:
                if src is not dst:
                    rows = slice(src.w_begin, src.w_begin + src.w_local)
                    dst.worker_bits[rows, a:b].copy_(src.worker_bits[rows, a:b])

    def _gather_rows(self, attr: str) -> None:
        for dst in self.ranks:
            for src in self.ranks:
                if src is not dst:
                    rows = slice(src.w_begin, src.w_begin + src.w_local)
                    getattr(dst, attr)[rows].copy_(getattr(src, attr)[rows])

    def _gather_ranges(self, attr: str, ranges_attr: str) -> None:
        for src in self.ranks:
            a, b = getattr(src, ranges_attr)[src.rank]
            if b <= a:
                continue
            for dst in self.ranks:
                if dst is not src:
                    getattr(dst, attr)[a:b].copy_(getattr(src, attr)[a:b])

    def step(self, all_grads: torch.Tensor) -> None:
        """all_grads: [W, n_padded]; rank r gets its workers' rows."""
        for r in self.ranks:
            r.worker_stage([all_grads[r.w_begin + i] for i in range(r.w_local)])
        if self.G > 1:
            if not self.peer_words:
                self._send_worker_chunks()
            self._gather_rows("worker_scales")
        for r in self.ranks:
            r.server_stage()
        if self.G > 1:
            if not self.peer_words:
                self._gather_ranges("server_bits", "word_ranges")
            self._gather_ranges("server_scales", "chunk_ranges")
        for r in self.ranks:
            r.apply_update()

    def close(self) -> None:
        for r in self.ranks:
            r.close()
