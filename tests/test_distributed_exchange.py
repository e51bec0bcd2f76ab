"""The split step's exchanges, on the CPU.

* The sums are exact: with each chunk's server words and scale computed by
  its owner and zeros elsewhere (what ob_server_stage leaves on a process),
  the sum over processes is the single-process result.  Checked with the
  oracle's per-chunk server stage, for ragged tensors and empty chunks.
* TorchExchange over world_size-2 gloo ranks: the in-place all-gather of
  row blocks and the sum-all-reduce of 32-bit words (bit 31 set included)
  and float scales.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle


def _owner_sums(n, W, G, seed):
    o = oracle.default()
    rng = np.random.default_rng(seed)
    bits = [rng.integers(0, 2**32, o.num_words(n), dtype=np.uint64).astype(np.uint32) for _ in range(W)]
    for b in bits:  # padding bits are 0
        if n % 32:
            b[-1] &= np.uint32((1 << (n % 32)) - 1)
    s = rng.uniform(0.5, 2.0, W).astype(np.float32)
    e0 = rng.normal(0, 0.1, n).astype(np.float32)
    # one process serving every chunk
    e_full = e0.copy()
    words_full, s_full = o.server_compress(bits, s, e_full)
    # G processes, each serving the chunks j % G == r, zeros elsewhere
    words_sum = np.zeros(o.num_words(n), np.int64)
    s_sum = np.zeros(W, np.float32)
    for r in range(G):
        e_r = e0.copy()
        words_r = np.zeros(o.num_words(n), np.uint32)
        s_r = np.zeros(W, np.float32)
        for j in range(W):
            if j % G == r:
                s_r[j] = o.server_compress_chunk(j, bits, s, e_r, words_r)
        words_sum += words_r.view(np.int32).astype(np.int64)
        s_sum = s_sum + s_r
        for j in range(W):  # each process's server error is right on its own chunks
            if j % G == r:
                b, e = o.chunk_range(n, W, j)
                np.testing.assert_array_equal(e_r[b:e], e_full[b:e])
    return words_full, s_full, words_sum, s_sum


@pytest.mark.parametrize("n,W,G", [(1 << 16, 8, 8), (100_003, 8, 4), (4097, 6, 3), (100, 16, 4),
                                   (33, 4, 2), (0, 4, 2)])
def test_owner_sums_equal_one_server(n, W, G):
    words_full, s_full, words_sum, s_sum = _owner_sums(n, W, G, seed=n + W + G)
    # 32-bit integer sums with one non-zero term per word: no carries
    assert np.array_equal(words_sum.astype(np.int32).view(np.uint32), words_full)
    assert np.array_equal(s_sum, s_full)


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
        words = torch.zeros(8, dtype=torch.int32)
        words[rank::world] = torch.tensor([-7 - rank, 2**30 + rank, -(2**31), 5][:len(words[rank::world])],
                                          dtype=torch.int32)
        ex.sum_(words)
        scales = torch.zeros(4, dtype=torch.float32)
        scales[rank::world] = torch.tensor([0.1 + rank, 3e-7][:len(scales[rank::world])])
        ex.sum_(scales)
        out[rank] = (rows.tolist(), words.tolist(), scales.tolist())
    finally:
        dist.destroy_process_group()


def test_torch_exchange_on_two_gloo_ranks():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == res[1]
    rows, words, scales = res[0]
    for q in range(world):
        blk = (np.arange(10).reshape(2, 5) + 100 * q).tolist()
        blk[0][0] = -(2**31) + q
        assert rows[2 * q:2 * q + 2] == blk
    assert words == [-7, -8, 2**30, 2**30 + 1, -(2**31), -(2**31), 5, 5]
    assert scales == [np.float32(0.1).item(), np.float32(1.1).item(),
                      np.float32(3e-7).item(), np.float32(3e-7).item()]


def test_worker_split_must_divide_W():
    from error_compensated_bit_adam_b200.distributed import DistributedOneBitAdam
    with pytest.raises(ValueError):
        DistributedOneBitAdam([10], 6, rank=0, world=4)
    with pytest.raises(ValueError):
        DistributedOneBitAdam([10], 4, rank=2, world=2)
