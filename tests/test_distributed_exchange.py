"""The split step's host logic on the CPU.

* ob_server_shard_range: the shards are contiguous, cover every server
  chunk and word exactly once, agree with ob_chunk_range's element ranges,
  and hold about the same number of tiles.
* The sums are exact: each shard's server words and scales (the oracle's
  per-chunk server stage on the shard's chunks, zeros elsewhere) summed
  over the shards equal the one-server result, bit for bit.
* TorchExchange over world_size-2 gloo ranks: the in-place all-gather of
  each rank's block of worker rows and the sum-all-reduce of zero-padded
  32-bit words (bit 31 set included) and float scales.
* The argument checks of DistributedOneBitAdam that need no GPU.
* The split step's whole protocol on two gloo ranks, the oracle doing each
  rank's arithmetic and TorchExchange and the shard ranges the exchange:
  bit for bit the single-process oracle run.
* A rank that leaves between steps is noticed at the next exchange."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from error_compensated_bit_adam_b200 import _binding as B

TILE = 4096


def _tiles_of_chunk(n, W, j):
    b, e = B.ob_chunk_range(n, W, j)
    return -(-(e - b) // TILE)


@pytest.mark.parametrize("numel,W,G", [([335544320], 8, 8), ([100_003, 31, 0, 4097, 70_000], 8, 4),
                                       ([50_001, 129, 12_345], 6, 3), ([100, 33, 5000], 16, 4),
                                       ([0, 0], 4, 3), ([1 << 20] * 5 + [7], 4, 8), ([33], 4, 1)])
def test_server_shards_partition_chunks_and_words(numel, W, G):
    offsets, n_pad = B.ob_layout(numel)
    C = len(numel) * W
    shards = [B.ob_server_shard_range(numel, W, G, r) for r in range(G)]
    assert shards[0][0] == 0 and shards[-1][1] == C
    assert shards[0][2] == 0 and shards[-1][3] == n_pad // 32
    for a, b in zip(shards, shards[1:]):
        assert a[1] == b[0] and a[3] == b[2]          # contiguous, no gap or overlap
    for cb, ce, wb, we in shards:
        assert cb <= ce and wb <= we
        # every real word of a served chunk lies in the shard's word range
        for c in range(cb, ce):
            t, j = divmod(c, W)
            b, e = B.ob_chunk_range(numel[t], W, j)
            if e > b:
                assert wb <= (offsets[t] + b) // 32 and (offsets[t] + e + 31) // 32 <= we
    tiles = [sum(_tiles_of_chunk(numel[c // W], W, c % W) for c in range(cb, ce))
             for cb, ce, _, _ in shards]
    biggest_chunk = max([_tiles_of_chunk(numel[c // W], W, c % W) for c in range(C)] + [0])
    assert max(tiles) - min(tiles) <= 2 * biggest_chunk + 1
    with pytest.raises(B.OnebitError):
        B.ob_server_shard_range(numel, W, G, G)


def _shard_sums(numel, W, G, seed):
    """One tensor list's server stage computed whole and per shard (the
    oracle's per-chunk server stage on the shard's chunks, zeros in the
    words and scales of the others), summed over the shards."""
    import oracle
    o = oracle.default()
    rng = np.random.default_rng(seed)
    shards = [B.ob_server_shard_range(numel, W, G, r) for r in range(G)]
    for t, n in enumerate(numel):
        bits = [rng.integers(0, 2**32, o.num_words(n), dtype=np.uint64).astype(np.uint32)
                for _ in range(W)]
        if n % 32:
            for b in bits:  # padding bits are 0
                b[-1] &= np.uint32((1 << (n % 32)) - 1)
        s = rng.uniform(0.5, 2.0, W).astype(np.float32)
        e0 = rng.normal(0, 0.1, n).astype(np.float32)
        e_one = e0.copy()
        words_one, s_one = o.server_compress(bits, s, e_one)
        words_sum = np.zeros(o.num_words(n), np.int64)
        s_sum = np.zeros(W, np.float32)
        for cb, ce, _, _ in shards:
            e_r = e0.copy()
            words_r = np.zeros(o.num_words(n), np.uint32)
            s_r = np.zeros(W, np.float32)
            for j in range(W):
                if cb <= t * W + j < ce:
                    s_r[j] = o.server_compress_chunk(j, bits, s, e_r, words_r)
                    b, e = o.chunk_range(n, W, j)
                    np.testing.assert_array_equal(e_r[b:e], e_one[b:e])  # server error on its shard
            words_sum += words_r.view(np.int32).astype(np.int64)
            s_sum = s_sum + s_r
        yield words_one, s_one, words_sum, s_sum


@pytest.mark.parametrize("numel,W,G", [([1 << 16], 8, 8), ([100_003, 31, 0, 4097, 70_000], 8, 4),
                                       ([50_001, 129, 12_345], 6, 3), ([100, 33, 5000], 16, 4),
                                       ([33], 4, 2)])
def test_shard_sums_equal_one_server(numel, W, G):
    for words_one, s_one, words_sum, s_sum in _shard_sums(numel, W, G, seed=W * G + len(numel)):
        # 32-bit integer sums with one non-zero term per word: no carries
        assert np.array_equal(words_sum.astype(np.int32).view(np.uint32), words_one)
        assert np.array_equal(s_sum, s_one)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    from error_compensated_bit_adam_b200.distributed import TorchExchange
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ex = TorchExchange()
        W, k = 2 * world, 5
        rows = torch.full((W, k), -1, dtype=torch.int32)
        rows[2 * rank:2 * rank + 2] = torch.arange(2 * k, dtype=torch.int32).view(2, k) + 100 * rank
        rows[2 * rank, 0] = -(2**31) + rank  # bit 31 set
        ex.gather_rows(rows, 2 * rank, 2)
        scales = torch.full((W, 3), -1.0, dtype=torch.float32)
        scales[2 * rank:2 * rank + 2] = 0.5 + rank
        ex.gather_rows(scales, 2 * rank, 2)
        words = torch.zeros(8, dtype=torch.int32)      # each word written by one rank
        words[rank::world] = torch.tensor([-7 - rank, 2**30 + rank, -(2**31), 5], dtype=torch.int32)
        ex.sum_(words)
        sp = torch.zeros(4, dtype=torch.float32)
        sp[rank::world] = torch.tensor([0.1 + rank, 3e-7])
        ex.sum_(sp)
        # per-chunk worker words: rank 0 serves columns [0, 6), rank 1 none
        chunk_rows = torch.full((W, 8), -1, dtype=torch.int32)
        chunk_rows[2 * rank:2 * rank + 2] = (torch.arange(16, dtype=torch.int32).view(2, 8)
                                             + 1000 * rank)
        ex.send_worker_chunks(chunk_rows, 2, [(0, 6), (6, 6)])
        # server ranges: rank 0 holds [0, 3), rank 1 [3, 7); [7, 9) is nobody's
        srv = torch.full((9,), -5.0)
        a, b = [(0, 3), (3, 7)][rank]
        srv[a:b] = torch.arange(a, b, dtype=torch.float32) + 0.25
        ex.gather_ranges(srv, [(0, 3), (3, 7)])
        out[rank] = (rows.tolist(), scales.tolist(), words.tolist(), sp.tolist(),
                     chunk_rows.tolist(), srv.tolist())
    finally:
        dist.destroy_process_group()


def test_torch_exchange_on_two_gloo_ranks():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][:4] == res[1][:4]
    rows, scales, words, sp, _, _ = res[0]
    for r in range(world):
        chunk_rows, srv = res[r][4], res[r][5]
        assert srv == [0.25, 1.25, 2.25, 3.25, 4.25, 5.25, 6.25, -5.0, -5.0]
        for q in range(world):
            for i in range(2):
                w = 2 * q + i
                want = [v + 1000 * q for v in range(8 * i, 8 * i + 8)]
                if q == r:
                    assert chunk_rows[w] == want            # own rows untouched
                elif r == 0:
                    assert chunk_rows[w] == want[:6] + [-1, -1]   # only rank 0's columns came
                else:
                    assert chunk_rows[w] == [-1] * 8       # rank 1 serves nothing
    assert words == [-7, -8, 2**30, 2**30 + 1, -(2**31), -(2**31), 5, 5]
    assert sp == [np.float32(0.1).item(), np.float32(1.1).item(),
                  np.float32(3e-7).item(), np.float32(3e-7).item()]
    for q in range(world):
        blk = (np.arange(10).reshape(2, 5) + 100 * q).tolist()
        blk[0][0] = -(2**31) + q
        assert rows[2 * q:2 * q + 2] == blk
        assert scales[2 * q:2 * q + 2] == [[0.5 + q] * 3] * 2


def test_worker_split_must_divide_W():
    from error_compensated_bit_adam_b200.distributed import DistributedOneBitAdam
    with pytest.raises(ValueError):
        DistributedOneBitAdam([10], 6, rank=0, world=4)
    with pytest.raises(ValueError):
        DistributedOneBitAdam([10], 4, rank=2, world=2)


def _rank_leaves(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    from error_compensated_bit_adam_b200.distributed import TorchExchange
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    ex = TorchExchange()
    rows = torch.zeros((2 * world, 4), dtype=torch.int32)
    ex.gather_rows(rows, 2 * rank, 2)                  # one step's exchange together
    dist.barrier()
    if rank == 1:
        out[rank] = "left"                              # leaves between steps, nothing in flight
        os._exit(0)
    try:
        ex.gather_rows(rows, 2 * rank, 2)              # the next step's exchange
        out[rank] = "no error"
    except Exception as e:  # the group's timeout or the closed connection
        out[rank] = f"error: {type(e).__name__}"
    os._exit(0)


def test_a_rank_that_leaves_is_detected_at_the_next_exchange():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_leaves, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res[1] == "left"
    assert res[0].startswith("error"), res[0]


def _grads(numel, W, step):
    rng = np.random.default_rng(1000 + step)
    return [[rng.normal(0, 1e-3, n).astype(np.float32) for n in numel] for _ in range(W)]


def _protocol_rank(rank, world, port, out, numel, W, steps):
    """One process of the split step with the oracle doing its arithmetic,
    on buffers in the library's padded layout: worker stage of its workers,
    the per-chunk exchange of the worker words (plus the worker scales),
    server stage of its shard, the exchange of the server words and scales,
    update of everything."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import oracle
    from error_compensated_bit_adam_b200.distributed import TorchExchange, exchange_plan
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ex = TorchExchange()
        hp = dict(beta1=0.9, beta2=0.999, eps=1e-8, lr=1e-4)
        params = [np.random.default_rng(7 + t).normal(0, 0.02, n).astype(np.float32)
                  for t, n in enumerate(numel)]
        run = oracle.OracleRun(params, W, hp)          # this process's state
        o, T, wl = run.o, len(numel), W // world
        mine = range(rank * wl, (rank + 1) * wl)
        offsets, n_pad = B.ob_layout(numel)
        chunk_ranges, word_ranges = exchange_plan(numel, W, world)
        cb, ce = chunk_ranges[rank]
        first = [off // 32 for off in offsets]
        nw = [o.num_words(n) for n in numel]
        received = 0
        for step in range(2):
            run.warmup_step(_grads(numel, W, step))    # every process, every worker
        run.freeze()
        for step in range(2, 2 + steps):
            g = _grads(numel, W, step)
            bits = torch.zeros((W, n_pad // 32), dtype=torch.int32)   # stale rows stay 0
            scales = torch.zeros((W, T), dtype=torch.float32)
            for w in mine:
                for t in range(T):
                    b, s = run.worker_stage(w, t, g[w][t])
                    bits[w, first[t]:first[t] + nw[t]] = torch.from_numpy(b.view(np.int32))
                    scales[w, t] = float(s)
            ex.send_worker_chunks(bits, wl, word_ranges)
            ex.gather_rows(scales, rank * wl, wl)
            sbits = torch.zeros(n_pad // 32, dtype=torch.int32)
            s_srv = torch.zeros(T * W, dtype=torch.float32)
            for t in range(T):
                rows = [bits[w, first[t]:first[t] + nw[t]].numpy().view(np.uint32).copy()
                        for w in range(W)]
                words_t = np.zeros(nw[t], np.uint32)
                for j in range(W):
                    if cb <= t * W + j < ce:
                        s_srv[t * W + j] = float(o.server_compress_chunk(
                            j, rows, scales[:, t].numpy(), run.e_s[t], words_t))
                sbits[first[t]:first[t] + nw[t]] = torch.from_numpy(words_t.view(np.int32))
            mine_words = sbits[slice(*word_ranges[rank])].clone()
            ex.gather_ranges(sbits, word_ranges)
            ex.gather_ranges(s_srv, chunk_ranges)
            assert torch.equal(sbits[slice(*word_ranges[rank])], mine_words)
            received += sum(b - a for q, (a, b) in enumerate(word_ranges) if q != rank)
            for t in range(T):
                full = sbits[first[t]:first[t] + nw[t]].numpy().view(np.uint32)
                for j in range(W):
                    o.apply_chunk(j, W, hp["lr"], full, s_srv[t * W + j].item(), run.d[t], run.p[t],
                                  run.m[t])
        served = {(t, j) for t in range(T) for j in range(W) if cb <= t * W + j < ce}
        out[rank] = ([p.tobytes() for p in run.p], [m.tobytes() for m in run.m],
                     {w: [e.tobytes() for e in run.e_w[w]] for w in mine},
                     {(t, j): run.e_s[t][slice(*o.chunk_range(numel[t], W, j))].tobytes()
                      for (t, j) in served}, received)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("numel,W,world", [([5_001, 64, 0, 777], 4, 2), ([70_000, 33], 6, 3),
                                           ([100, 33, 5000], 8, 4)])
def test_split_protocol_on_gloo_ranks_equals_one_process(numel, W, world):
    import oracle
    steps = 3
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_protocol_rank, args=(world, _free_port(), out, numel, W, steps), nprocs=world,
                 join=True)
        res = dict(out)
    hp = dict(beta1=0.9, beta2=0.999, eps=1e-8, lr=1e-4)
    params = [np.random.default_rng(7 + t).normal(0, 0.02, n).astype(np.float32)
              for t, n in enumerate(numel)]
    ref = oracle.OracleRun(params, W, hp)
    for step in range(2):
        ref.warmup_step(_grads(numel, W, step))
    ref.freeze()
    for step in range(2, 2 + steps):
        ref.compressed_step(_grads(numel, W, step))
    o = ref.o
    n_words = B.ob_layout(numel)[1] // 32
    for r in range(world):
        p, m, e_w, e_s, received = res[r]
        assert received < steps * n_words      # only the other ranks' words came in
        assert p == [a.tobytes() for a in ref.p] and m == [a.tobytes() for a in ref.m]
        for w, rows in e_w.items():
            assert rows == [e.tobytes() for e in ref.e_w[w]]
        for (t, j), blob in e_s.items():
            assert blob == ref.e_s[t][slice(*o.chunk_range(numel[t], W, j))].tobytes()
    served = set().union(*(set(res[r][3]) for r in range(world)))
    assert served == {(t, j) for t in range(len(numel)) for j in range(W)}
