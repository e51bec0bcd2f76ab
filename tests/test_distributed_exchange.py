"""The split step's exchange on the CPU: TorchExchange over world_size-2
gloo ranks (the in-place all-gather of each rank's block of worker rows,
32-bit words with bit 31 set included), and the argument checks of
DistributedOneBitAdam that need no GPU."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


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
        out[rank] = (rows.tolist(), scales.tolist())
    finally:
        dist.destroy_process_group()


def test_torch_exchange_on_two_gloo_ranks():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == res[1]
    rows, scales = res[0]
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
