"""The split step (ob_worker_stage / ob_server_stage / ob_apply_update with
the exchanges between them) against one ob_compressed_step context.

G ranks run in one process on one GPU (distributed.LocalRanks), each with
its own context and its own range of server chunks, the exchanges done by
device copies of the ranges the processes would send each other.  The bar
is bit for bit: parameters, momentum, the server words and scales, every
worker scale on every rank, each rank's own workers' words whole and the
other workers' words over the chunks the rank serves, the worker errors on
their rank and the server error on the rank serving each chunk, after
warmup, freeze and several compressed steps with fresh gradients.  The
same runs are also compared with the CPU oracle."""
import numpy as np
import pytest
import torch

from error_compensated_bit_adam_b200 import _binding as B
from error_compensated_bit_adam_b200 import workloads as WL
from error_compensated_bit_adam_b200.distributed import DistributedOneBitAdam, LocalRanks
from error_compensated_bit_adam_b200.optimizer import OneBitAdam
import oracle

pytestmark = pytest.mark.gpu

CASES = {
    # (tensor sizes, W, G)
    "flat-W8-G8": ((1 << 18,), 8, 8),
    "flat-W8-G2": ((1 << 18,), 8, 2),
    "ragged-W8-G4": ((100_003, 31, 0, 4097, 70_000), 8, 4),
    "ragged-W6-G3": ((50_001, 129, 12_345), 6, 3),
    "empty-chunks-W16-G4": ((100, 33, 5000), 16, 4),
    "W4-G1": ((30_000, 7), 4, 1),
    "ragged-W8-G8": ((100_003, 31, 0, 4097, 70_000, 1 << 16), 8, 8),
    "two-tensors-W4-G2": ((4096 * 5 + 17, 4096 * 3), 4, 2),
}


def _run(sizes, W, G, warmup=2, compressed=4, seed=31, orc=False, peer_words=False):
    wl = WL.Workload(f"split-{W}-{G}", tuple((n,) for n in sizes), W, warmup, compressed, seed=seed,
                     zero_fraction=0.2)
    offsets, n_pad = B.ob_layout(wl.numels)
    params = WL.make_params(wl, offsets, n_pad, device="cuda")
    scale = WL.grad_scale_vector(wl, offsets, n_pad, device="cuda")
    ref = OneBitAdam(wl.numels, W, params=params.clone(), **WL.HYPER)
    ranks = LocalRanks(wl.numels, W, G, peer_words=peer_words, **WL.HYPER)
    run = (oracle.OracleRun(WL.split(params.cpu().numpy(), offsets, wl.numels), W, WL.HYPER)
           if orc else None)
    for r in ranks.ranks:
        r.params.copy_(params)
    g = torch.empty((W, n_pad), device="cuda")

    def host(g):
        h = g.cpu().numpy()
        return [WL.split(h[w], offsets, wl.numels) for w in range(W)]

    step = 0
    for _ in range(warmup):
        WL.fill_grads(wl, step, scale, g)
        step += 1
        ref.warmup_step(g)
        ranks.warmup_step(g)
        if run:
            run.warmup_step(host(g))
    ref.freeze()
    ranks.freeze()
    if run:
        run.freeze()
    for _ in range(compressed):
        WL.fill_grads(wl, step, scale, g)
        step += 1
        ref.step(g)
        ranks.step(g)
        if run:
            run.compressed_step(host(g))
    torch.cuda.synchronize()
    return (ref, ranks, run) if orc else (ref, ranks)


@pytest.mark.parametrize("peer_words", [False, True], ids=["exchange", "peer-words"])
@pytest.mark.parametrize("name", list(CASES))
def test_split_step_equals_one_context(name, peer_words):
    """Both forms of the word exchanges: by the caller (device copies of
    the ranges, as NCCL moves them between processes), and inside the
    kernels (the worker stage storing into the serving rank's rows, the
    update reading the serving rank's words; here the "peers" are the other
    contexts' buffers on the same GPU)."""
    sizes, W, G = CASES[name]
    ref, ranks = _run(sizes, W, G, peer_words=peer_words)
    try:
        want = {k: ref.read(k) for k in (B.OB_STATE_P, B.OB_STATE_M, B.OB_STATE_BITS_SERVER,
                                          B.OB_STATE_S_SERVER, B.OB_STATE_S_WORKER, B.OB_STATE_STEP)}
        want_bits = [ref.read(B.OB_STATE_BITS_WORKER, w) for w in range(W)]
        for r in ranks.ranks:
            for k, v in want.items():
                np.testing.assert_array_equal(r.read(k), v, err_msg=f"{name} rank {r.rank} kind {k}")
            a, b = r.word_ranges[r.rank]             # the words of the chunks r serves
            for w in range(W):
                got = r.read(B.OB_STATE_BITS_WORKER, w)
                if r.w_begin <= w < r.w_begin + r.w_local and not peer_words:
                    np.testing.assert_array_equal(got, want_bits[w])
                else:  # with peer words a rank's own words of other chunks went to their servers
                    np.testing.assert_array_equal(got[a:b], want_bits[w][a:b])
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


@pytest.mark.parametrize("sizes,W,G", [((1 << 18,), 8, 2), ((100_003, 31, 0, 4097, 70_000), 8, 4),
                                       ((100, 33, 5000), 16, 8), ((50_001, 129, 12_345), 6, 3)])
def test_split_step_follows_the_oracle(sizes, W, G):
    """The split step against the CPU oracle over the same schedule: worker
    and server scales within 1e-6 relative, the server words bit for bit
    while every scale has matched the oracle's exactly (else at most 1e-3
    of the bits), parameters within 1e-5 relative L2 after 4 free-running
    compressed steps."""
    ref, ranks, run = _run(sizes, W, G, orc=True)
    try:
        offsets, _ = ref.layout()
        for r in ranks.ranks:
            s_w = r.read(B.OB_STATE_S_WORKER)
            s_s = r.read(B.OB_STATE_S_SERVER)
            np.testing.assert_allclose(s_w, run.s_w, rtol=1e-6, atol=0)
            np.testing.assert_allclose(s_s, run.s_srv, rtol=1e-6, atol=0)
            words = r.read(B.OB_STATE_BITS_SERVER)
            exact = np.array_equal(s_w, run.s_w) and np.array_equal(s_s, run.s_srv)
            for t, n in enumerate(sizes):
                got = words[offsets[t] // 32:offsets[t] // 32 + (n + 31) // 32]
                diff = int(np.unpackbits((got ^ run.sbits[t]).view(np.uint8)).sum())
                assert diff == 0 or (not exact and diff <= max(1, 1e-3 * 32 * got.size)), (t, diff)
            p = np.concatenate(WL.split(r.read(B.OB_STATE_P), offsets, list(sizes))).astype(np.float64)
            want = np.concatenate(run.p).astype(np.float64)
            assert np.linalg.norm(p - want) <= 1e-5 * np.linalg.norm(want)
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
        bits = opt.worker_bits.data_ptr()
        sbits = opt.server_bits.data_ptr()
        for bad, status in ((([bits], [sbits]), B.OB_ERR_INVALID_ARG),       # one shard of two
                            (([bits, 0], [sbits, sbits]), B.OB_ERR_INVALID_ARG),
                            (([bits, bits + 4], [sbits, sbits]), B.OB_ERR_ALIGN)):
            with pytest.raises(B.OnebitError) as e:
                B.ob_set_peer_words(ctx, *bad)
            assert e.value.status == status
        B.ob_set_peer_words(ctx, [bits, bits], [sbits, sbits])
        with pytest.raises(B.OnebitError) as e:
            B.ob_set_server_shard(ctx, 1, 0)                   # peers were set for two shards
        assert e.value.status == B.OB_ERR_PHASE
        B.ob_set_peer_words(ctx, [], [])                       # off again
        B.ob_set_server_shard(ctx, 1, 0)                       # serve everything again
        B.ob_worker_stage(ctx, [0, 0, 0, 0], 0, 0)             # an empty range is a no-op stage
        B.ob_server_stage(ctx)
        B.ob_apply_update(ctx)
        assert opt.read(B.OB_STATE_STEP)[1] == 2
    finally:
        opt.close()
