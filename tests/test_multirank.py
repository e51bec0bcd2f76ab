"""The multi-GPU host logic of bench.py, on CPU ranks over gloo.

bench.py --gpus N runs N independent replicas (the method's exchange lives
inside one GPU's HBM), so the only cross-rank logic is the barrier around
the timed region, the max of the step times over ranks and the whole-job
aggregate.  These run here as world_size-2 gloo ranks; no GPU is used."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [4.0, 7.5][rank]           # rank 1 is the slow one
        bench.barrier(world)
        ms = bench.max_over_ranks(local_ms, world)
        value = bench.replica_throughput(1000, world, ms)
        out[rank] = (ms, value)
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_step_and_sum_replicas():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == res[1]                   # every rank sees the same numbers
    ms, value = res[0]
    assert ms == 7.5
    assert value == pytest.approx(2 * 1000 / 7.5e-3)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.0, 1) == 3.0
    bench.barrier(1)
    assert bench.replica_throughput(10, 1, 2.0) == pytest.approx(5000.0)


class _FakeOpt:
    """Stands in for OneBitAdam in the end-to-end leg: step_host fails on
    the rank told to."""

    def __init__(self, fail):
        self.fail = fail

    def step_host(self, host, out):
        if self.fail:
            raise RuntimeError("injected on the host")


def _e2e_rank(rank, world, port, out, fail_rank):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    import types
    import bench
    from error_compensated_bit_adam_b200 import workloads as WL
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    try:
        wl = WL.flat(1000, 2, 1, 1, seed=1, name="e2e-fake")
        args = types.SimpleNamespace(steps=3, e2e_steps=2)
        res = bench.measure_e2e(_FakeOpt(rank == fail_rank), wl, 1024, torch.zeros((2, 1024)), args,
                                world, "cpu")
        out[rank] = res
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_e2e_leg_takes_the_same_collectives_when_one_rank_fails():
    world = 2
    for fail_rank in (-1, 1):
        with mp.Manager() as mgr:
            out = mgr.dict()
            mp.spawn(_e2e_rank, args=(world, _free_port(), out, fail_rank), nprocs=world, join=True)
            res = dict(out)
        if fail_rank < 0:
            assert res[0]["value"] is not None and res[0]["value"] == res[1]["value"]
        else:
            assert res[0]["value"] is None and res[1]["value"] is None
            assert "injected" in res[1]["error"] and res[0]["error"] == "failed on another rank"
