"""The split step (ob_worker_stage / ob_server_stage / ob_apply_update with
the exchanges between them) against one ob_compressed_step context.

G ranks run in one process on one GPU (distributed.LocalRanks), each with
its own context and its own range of server chunks, the exchanges done by
device copies and sums.  The bar is bit for bit: parameters, momentum, the
server words and scales, and every worker's words and scales on every
rank, the worker errors on their rank and the server error on the rank
serving each chunk, after warmup, freeze and several compressed steps with
fresh gradients."""
import numpy as np
import pytest
import torch

from error_compensated_bit_adam_b200 import _binding as B
from error_compensated_bit_adam_b200 import workloads as WL
from error_compensated_bit_adam_b200.distributed import DistributedOneBitAdam, LocalRanks
from error_compensated_bit_adam_b200.optimizer import OneBitAdam

pytestmark = pytest.mark.gpu

CASES = {
    # (tensor sizes, W, G)
    "flat-W8-G8": ((1 << 18,), 8, 8),
    "flat-W8-G2": ((1 << 18,), 8, 2),
    "ragged-W8-G4": ((100_003, 31, 0, 4097, 70_000), 8, 4),
    "ragged-W6-G3": ((50_001, 129, 12_345), 6, 3),
    "empty-chunks-W16-G4": ((100, 33, 5000), 16, 4),
    "W4-G1": ((30_000, 7), 4, 1),
}


def _run(sizes, W, G, warmup=2, compressed=4, seed=31):
    wl = WL.Workload(f"split-{W}-{G}", tuple((n,) for n in sizes), W, warmup, compressed, seed=seed,
                     zero_fraction=0.2)
    offsets, n_pad = B.ob_layout(wl.numels)
    params = WL.make_params(wl, offsets, n_pad, device="cuda")
    scale = WL.grad_scale_vector(wl, offsets, n_pad, device="cuda")
    ref = OneBitAdam(wl.numels, W, params=params.clone(), **WL.HYPER)
    ranks = LocalRanks(wl.numels, W, G, **WL.HYPER)
    for r in ranks.ranks:
        r.params.copy_(params)
    g = torch.empty((W, n_pad), device="cuda")
    step = 0
    for _ in range(warmup):
        WL.fill_grads(wl, step, scale, g)
        step += 1
        ref.warmup_step(g)
        ranks.warmup_step(g)
    ref.freeze()
    ranks.freeze()
    for _ in range(compressed):
        WL.fill_grads(wl, step, scale, g)
        step += 1
        ref.step(g)
        ranks.step(g)
    torch.cuda.synchronize()
    return ref, ranks


@pytest.mark.parametrize("name", list(CASES))
def test_split_step_equals_one_context(name):
    sizes, W, G = CASES[name]
    ref, ranks = _run(sizes, W, G)
    try:
        want = {k: ref.read(k) for k in (B.OB_STATE_P, B.OB_STATE_M, B.OB_STATE_BITS_SERVER,
                                          B.OB_STATE_S_SERVER, B.OB_STATE_S_WORKER, B.OB_STATE_STEP)}
        want_bits = [ref.read(B.OB_STATE_BITS_WORKER, w) for w in range(W)]
        for r in ranks.ranks:
            for k, v in want.items():
                np.testing.assert_array_equal(r.read(k), v, err_msg=f"{name} rank {r.rank} kind {k}")
            for w in range(W):
                np.testing.assert_array_equal(r.read(B.OB_STATE_BITS_WORKER, w), want_bits[w])
            for w in range(r.w_begin, r.w_begin + r.w_local):  # errors live with their worker
                np.testing.assert_array_equal(r.read(B.OB_STATE_E_WORKER, w),
                                              ref.read(B.OB_STATE_E_WORKER, w))
        # the server error of a chunk lives on the rank serving it
        e_ref = ref.read(B.OB_STATE_E_SERVER)
        offsets, _ = ref.layout()
        served = 0
        for rk in ranks.ranks:
            e = rk.read(B.OB_STATE_E_SERVER)
            for t, n in enumerate(sizes):
                for j in range(W):
                    if rk.serves(t, j):
                        served += 1
                        b, end = B.ob_chunk_range(n, W, j)
                        np.testing.assert_array_equal(e[offsets[t] + b:offsets[t] + end],
                                                      e_ref[offsets[t] + b:offsets[t] + end])
        assert served == len(sizes) * W
    finally:
        ref.close()
        ranks.close()


@pytest.mark.parametrize("G", [1, 2, 4])
def test_allreduce_warmup_matches_the_ordered_warmup(G):
    """The warmup on all-reduced sums: bit for bit with one rank (the sums
    are the gradients themselves), within rounding of the sum's order
    otherwise; the compressed steps after it still track one context."""
    sizes, W = (100_003, 4097, 33), 4
    wl = WL.Workload("allreduce-warmup", tuple((n,) for n in sizes), W, 3, 4, seed=41)
    offsets, n_pad = B.ob_layout(wl.numels)
    params = WL.make_params(wl, offsets, n_pad, device="cuda")
    scale = WL.grad_scale_vector(wl, offsets, n_pad, device="cuda")
    ref = OneBitAdam(wl.numels, W, params=params.clone(), **WL.HYPER)
    ranks = LocalRanks(wl.numels, W, G, **WL.HYPER)
    try:
        for r in ranks.ranks:
            r.params.copy_(params)
        g = torch.empty((W, n_pad), device="cuda")
        for step in range(3):
            WL.fill_grads(wl, step, scale, g)
            ref.warmup_step(g)
            ranks.warmup_step_allreduce(g)
        ref.freeze()
        ranks.freeze()
        p_ref = ref.read(B.OB_STATE_P).astype(np.float64)
        for r in ranks.ranks:
            p = r.read(B.OB_STATE_P).astype(np.float64)
            if G == 1:
                np.testing.assert_array_equal(p, p_ref)
                np.testing.assert_array_equal(r.read(B.OB_STATE_D), ref.read(B.OB_STATE_D))
            else:
                assert np.linalg.norm(p - p_ref) <= 1e-6 * np.linalg.norm(p_ref)
        for step in range(3, 7):
            WL.fill_grads(wl, step, scale, g)
            ref.step(g)
            ranks.step(g)
        p_ref = ref.read(B.OB_STATE_P).astype(np.float64)
        for r in ranks.ranks:
            p = r.read(B.OB_STATE_P).astype(np.float64)
            assert np.linalg.norm(p - p_ref) <= 1e-5 * np.linalg.norm(p_ref)
    finally:
        ref.close()
        ranks.close()


def test_split_step_phase_rules():
    opt = DistributedOneBitAdam([4096], 4, rank=1, world=2, **WL.HYPER)
    try:
        ctx = opt.opt.ctx
        g = torch.zeros((4, 4096), device="cuda")
        ptrs = [0, 0, g[2].data_ptr(), g[3].data_ptr()]
        opt.warmup_step(g)
        for call in (lambda: B.ob_worker_stage(ctx, ptrs, 2, 2),  # before the freeze
                     lambda: B.ob_server_stage(ctx),
                     lambda: B.ob_apply_update(ctx)):
            with pytest.raises(B.OnebitError) as e:
                call()
            assert e.value.status == B.OB_ERR_PHASE
        opt.freeze()
        for bad in ((2, 3), (-1, 1)):                          # outside [0, W)
            with pytest.raises(B.OnebitError) as e:
                B.ob_worker_stage(ctx, ptrs, *bad)
            assert e.value.status == B.OB_ERR_INVALID_ARG
        with pytest.raises(B.OnebitError) as e:
            B.ob_worker_stage(ctx, [0, 0, 0, g[3].data_ptr()], 2, 2)  # a NULL gradient in range
        assert e.value.status == B.OB_ERR_INVALID_ARG
        opt.worker_stage([g[2], g[3]])
        for call in (lambda: B.ob_worker_stage(ctx, ptrs, 2, 2),
                     lambda: B.ob_apply_update(ctx),
                     lambda: B.ob_set_server_shard(ctx, 1, 0),
                     lambda: B.ob_compressed_step(ctx, [g[w].data_ptr() for w in range(4)]),
                     lambda: opt.opt.write(B.OB_STATE_P, 0, np.zeros(4096, np.float32)),
                     lambda: opt.warmup_step(g)):
            with pytest.raises(B.OnebitError) as e:
                call()
            assert e.value.status == B.OB_ERR_PHASE
        opt.read(B.OB_STATE_BITS_WORKER, 2)                     # reading is allowed
        opt.server_stage()
        with pytest.raises(B.OnebitError) as e:
            B.ob_server_stage(ctx)                             # twice
        assert e.value.status == B.OB_ERR_PHASE
        opt.apply_update()
        assert opt.read(B.OB_STATE_STEP)[1] == 1
        with pytest.raises(B.OnebitError) as e:
            B.ob_set_server_shard(ctx, 2, 2)                   # no such shard
        assert e.value.status == B.OB_ERR_INVALID_ARG
        B.ob_set_server_shard(ctx, 1, 0)                       # serve everything again
        B.ob_worker_stage(ctx, [0, 0, 0, 0], 0, 0)             # an empty range is a no-op stage
        B.ob_server_stage(ctx)
        B.ob_apply_update(ctx)
        assert opt.read(B.OB_STATE_STEP)[1] == 2
    finally:
        opt.close()
