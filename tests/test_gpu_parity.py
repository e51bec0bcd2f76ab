"""CUDA path (through the C ABI) against the CPU oracle.

Bar: warmup and freeze state bit for bit; packed sign words bit for bit;
scales within 1e-6 relative; in re-synced steps the new errors, momentum
and parameters bit for bit (when the scales agree exactly, which is the
rule); after 10 free-running steps parameters within 1e-5 relative L2.
"""
import numpy as np
import pytest
import torch

from error_compensated_bit_adam_b200 import _binding as B
from error_compensated_bit_adam_b200 import workloads as WL
from error_compensated_bit_adam_b200.optimizer import OneBitAdam
from gpu_harness import Pair, run_schedule

pytestmark = pytest.mark.gpu

PARAM_TOL = 1e-5


def small_encoder(W=16):
    return WL.Workload("encoder-2L-h64-W16", WL.encoder_shapes(2, 64, 256, 1000, 64), W, 3, 6, seed=21,
                       fan_in_scaling=True)


def small_ragged(W=8, count=120, max_log2=14):
    return WL.Workload("ragged-120-W8", WL.ragged_sizes(count, seed=22, max_log2=max_log2), W, 3, 6,
                       seed=22, zero_fraction=WL.ZERO_FRACTION)


CASES = {
    "flat-1M-W4": WL.FLAT_1M_W4,
    "encoder-small-W16": small_encoder(),
    "ragged-small-W8": small_ragged(),
    "flat-ragged-tail-W3": WL.flat(100_003, 3, 3, 5, seed=23),
    "flat-W5": WL.flat(40_000, 5, 2, 4, seed=24),
    "flat-W1": WL.flat(70_001, 1, 2, 4, seed=25),
    # W past the 8 tabulated workers, not a power of two (the server stage
    # adds workers 8.. one by one and divides by W)
    "flat-W9": WL.flat(90_001, 9, 2, 4, seed=30),
    "ragged-W12": WL.Workload("ragged-W12", ((50_000,), (4_097,), (0,), (33,)), 12, 2, 4, seed=31,
                              zero_fraction=0.1),
    # > 2048 tiles per tensor and per server chunk: multi-segment scale sums
    "flat-multi-segment-W2": WL.flat((1 << 24) + 12_345, 2, 1, 2, seed=29),
}


@pytest.mark.parametrize("name", list(CASES))
def test_resynced_steps_match_oracle_bit_for_bit(name):
    pr, flags = run_schedule(CASES[name], synced=True)
    try:
        assert sum(flags) >= len(flags) - 1, f"scales differed in the last ulp too often: {flags}"
    finally:
        pr.close()


@pytest.mark.parametrize("name", list(CASES))
def test_free_running_steps_stay_within_tolerance(name):
    pr, flags = run_schedule(CASES[name], synced=False)
    try:
        assert pr.params_rel_l2() <= PARAM_TOL
    finally:
        pr.close()


@pytest.mark.parametrize("W", [2, 8, 24, 32, 48, 64])
def test_sweep_small_n(W):
    wl = WL.flat(1 << 20, W, 2, 3, seed=26, name=f"sweep-small-W{W}")
    pr, flags = run_schedule(wl, synced=False)
    try:
        assert pr.params_rel_l2() <= PARAM_TOL
    finally:
        pr.close()


EDGE = {
    "single-element": ((1,), 4),
    "empty-tensors-around": ((0, 5, 0), 4),
    "one-word-minus-one": ((31,), 2),
    "one-word-plus-one": ((33,), 2),
    "pad-boundaries": ((127, 128, 129), 3),
    "fewer-words-than-servers": ((100,), 8),
    "many-workers-tiny": ((300, 7), 64),
    "tile-boundaries": ((4095, 4096, 4097, 8192 + 1), 2),
    # the server stage's table and 55 workers added one by one, W not a
    # power of two; and 17 workers over ragged tensors
    "workers-63": ((5_000, 33), 63),
    "workers-17-ragged": ((12_345, 4_097, 1, 0), 17),
}


@pytest.mark.parametrize("name", list(EDGE))
def test_edge_cases(name):
    shapes, W = EDGE[name]
    wl = WL.Workload(name, tuple((n,) for n in shapes), W, 2, 4, seed=27,
                     zero_fraction=0.2 if name == "pad-boundaries" else 0.0)
    pr, flags = run_schedule(wl, synced=True)
    pr.close()
    pr, flags = run_schedule(wl, synced=False)
    try:
        assert pr.params_rel_l2() <= PARAM_TOL
    finally:
        pr.close()


def test_all_empty_tensors_is_a_noop():
    opt = OneBitAdam([0, 0], 4, **WL.HYPER)
    g = torch.zeros((4, 0), device="cuda")
    opt.warmup_step(g)
    opt.freeze()
    opt.step(g)
    assert np.all(opt.read(B.OB_STATE_S_WORKER) == 0)
    assert np.all(opt.read(B.OB_STATE_S_SERVER) == 0)
    assert list(opt.read(B.OB_STATE_STEP)) == [1, 1, 1]
    opt.close()


def test_runs_are_deterministic():
    wl = small_ragged(W=4, count=40)
    outs = []
    for _ in range(2):
        pr = Pair(wl)
        for _ in range(2):
            pr.warmup_step()
        pr.freeze()
        for _ in range(3):
            pr.compressed_step()
        outs.append([pr.gpu.read(B.OB_STATE_P), pr.gpu.read(B.OB_STATE_S_SERVER),
                     pr.gpu.read(B.OB_STATE_BITS_SERVER), pr.gpu.read(B.OB_STATE_E_WORKER, 3)])
        pr.close()
    for a, b in zip(*outs):
        assert np.array_equal(a.view(np.uint8), b.view(np.uint8))


def test_host_gradients_path_matches_device_path():
    wl = WL.Workload("ragged-host", WL.ragged_sizes(60, seed=28, max_log2=20), 4, 2, 3, seed=28)
    a, b = Pair(wl), Pair(wl)
    try:
        for pr in (a, b):
            for _ in range(2):
                pr.warmup_step()
            pr.freeze()
        for _ in range(3):
            a.next_grads()
            a.gpu.step(a.grads)
            b.next_grads()
            host = b.grads.cpu().pin_memory()
            scales = np.zeros(len(wl.numels) * wl.W, np.float32)
            b.gpu.step_host(host, scales)
            assert np.array_equal(scales.reshape(-1, wl.W), b.gpu.read(B.OB_STATE_S_SERVER))
        for kind in (B.OB_STATE_P, B.OB_STATE_M, B.OB_STATE_E_SERVER):
            assert np.array_equal(a.gpu.read(kind).view(np.uint32), b.gpu.read(kind).view(np.uint32))
        for w in range(wl.W):
            assert np.array_equal(a.gpu.read(B.OB_STATE_E_WORKER, w), b.gpu.read(B.OB_STATE_E_WORKER, w))
    finally:
        a.close()
        b.close()


def test_phase_and_argument_errors():
    opt = OneBitAdam([1000, 10], 2, **WL.HYPER)
    n = opt.n_padded
    g = torch.zeros((2, n), device="cuda")
    ptrs = [g[0].data_ptr(), g[1].data_ptr()]

    def status(fn, *a):
        with pytest.raises(B.OnebitError) as ei:
            fn(*a)
        return ei.value.status

    assert status(B.ob_freeze_variance, opt.ctx) == B.OB_ERR_PHASE          # no warmup yet
    assert status(B.ob_compressed_step, opt.ctx, ptrs) == B.OB_ERR_PHASE     # not frozen
    assert status(B.ob_read_state, opt.ctx, B.OB_STATE_D, 0, 0, 1) == B.OB_ERR_INVALID_ARG
    buf = np.zeros(n, np.float32)
    assert status(B.ob_read_state, opt.ctx, B.OB_STATE_D, 0, buf.ctypes.data, buf.nbytes) == B.OB_ERR_PHASE
    assert status(B.ob_warmup_adam_step, opt.ctx, [ptrs[0] + 4, ptrs[1]]) == B.OB_ERR_ALIGN
    assert status(B.ob_warmup_adam_step, opt.ctx, [ptrs[0], 0]) == B.OB_ERR_INVALID_ARG
    opt.warmup_step(g)
    opt.freeze()
    assert status(B.ob_freeze_variance, opt.ctx) == B.OB_ERR_PHASE          # already frozen
    assert status(B.ob_warmup_adam_step, opt.ctx, ptrs) == B.OB_ERR_PHASE   # after freeze
    assert status(B.ob_read_state, opt.ctx, B.OB_STATE_V, 0, buf.ctypes.data, buf.nbytes) == B.OB_ERR_PHASE
    assert status(B.ob_read_state, opt.ctx, B.OB_STATE_E_WORKER, 2, buf.ctypes.data, buf.nbytes) == B.OB_ERR_INVALID_ARG
    assert status(B.ob_read_state, opt.ctx, B.OB_STATE_M, 0, buf.ctypes.data, buf.nbytes - 4) == B.OB_ERR_INVALID_ARG
    w = np.zeros(n // 32, np.uint32)
    assert status(B.ob_write_state, opt.ctx, B.OB_STATE_BITS_SERVER, 0, w.ctypes.data, w.nbytes) == B.OB_ERR_INVALID_ARG
    step = np.array([0, 0, 1], np.int64)
    assert status(B.ob_write_state, opt.ctx, B.OB_STATE_STEP, 0, step.ctypes.data, step.nbytes) == B.OB_ERR_INVALID_ARG
    opt.step(g)
    assert list(opt.read(B.OB_STATE_STEP)) == [1, 1, 1]
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    host = torch.zeros((2, n)).pin_memory()
    assert status(B.ob_compressed_step_host, opt.ctx, [host[0].data_ptr(), host[1].data_ptr()],
                  small.data_ptr(), 16, None) == B.OB_ERR_WORKSPACE
    ctx = opt.ctx
    opt.close()
    assert status(B.ob_compressed_step, ctx, ptrs) == B.OB_ERR_INVALID_ARG   # destroyed


def test_checkpoint_resume_through_state_io():
    """Read every writable piece of state, restore it into a fresh context,
    and continue: the two runs stay bit-identical."""
    wl = small_ragged(W=4, count=30)
    a = Pair(wl)
    for _ in range(2):
        a.warmup_step()
    a.freeze()
    a.compressed_step()
    saved = {k: a.gpu.read(k) for k in (B.OB_STATE_P, B.OB_STATE_M, B.OB_STATE_D,
                                        B.OB_STATE_E_SERVER, B.OB_STATE_STEP)}
    saved_e = [a.gpu.read(B.OB_STATE_E_WORKER, w) for w in range(wl.W)]
    b = OneBitAdam(wl.numels, wl.W, **WL.HYPER)
    b.write(B.OB_STATE_STEP, 0, saved[B.OB_STATE_STEP])
    for k in (B.OB_STATE_P, B.OB_STATE_M, B.OB_STATE_D, B.OB_STATE_E_SERVER):
        b.write(k, 0, saved[k])
    for w in range(wl.W):
        b.write(B.OB_STATE_E_WORKER, w, saved_e[w])
    for _ in range(2):
        a.next_grads()
        a.gpu.step(a.grads)
        b.step(a.grads)
    for k in (B.OB_STATE_P, B.OB_STATE_M, B.OB_STATE_E_SERVER, B.OB_STATE_BITS_SERVER,
              B.OB_STATE_S_SERVER, B.OB_STATE_STEP):
        assert np.array_equal(a.gpu.read(k), b.read(k)), k
    a.close()
    b.close()


def test_profiling_counters():
    wl = small_ragged(W=4, count=30)
    pr = Pair(wl)
    pr.gpu.profile(True)
    pr.warmup_step()
    pr.freeze()
    for _ in range(3):
        pr.compressed_step()
    prof = pr.gpu.profile_read(reset=True)
    assert prof["ob_warmup_kernel"][1] == 1 and prof["ob_freeze_kernel"][1] == 1
    for k in ("ob_pack_kernel", "ob_scale_kernel:worker", "ob_server_kernel",
              "ob_scale_kernel:server", "ob_apply_kernel"):
        assert prof[k][1] == 3 and prof[k][0] > 0, k
    assert all(v == (0.0, 0) for v in pr.gpu.profile_read().values())
    pr.close()


@pytest.mark.parametrize("hp", [dict(beta1=0.95, beta2=0.98, eps=1e-6, lr=3e-3),
                                dict(beta1=0.5, beta2=0.9, eps=1e-4, lr=0.05)],
                         ids=["b0.95-b0.98", "b0.5-b0.9"])
def test_other_hyperparameters(hp):
    wl = small_ragged(W=4, count=40)
    pr, flags = run_schedule(wl, synced=True, hp=hp)
    pr.close()
    pr, flags = run_schedule(wl, synced=False, hp=hp)
    try:
        assert pr.params_rel_l2() <= PARAM_TOL
    finally:
        pr.close()


def test_bucketed_contexts_on_two_streams_match_sequential():
    """Two parameter buckets, each its own context on its own stream (the
    way a trainer overlaps optimizer steps with backward), stepping
    concurrently, end bit-identical to the same buckets stepped one after
    the other."""
    buckets = [small_ragged(W=4, count=30), WL.flat(300_001, 4, 2, 3, seed=31)]
    dev = torch.device("cuda")

    def run(concurrent):
        streams = [torch.cuda.Stream() for _ in buckets]
        opts, grads = [], []
        for wl, st in zip(buckets, streams):
            offs, n_pad = B.ob_layout(wl.numels)
            params = WL.make_params(wl, offs, n_pad, device=dev)
            scale = WL.grad_scale_vector(wl, offs, n_pad, device=dev)
            g = torch.empty((wl.W, n_pad), device=dev)
            WL.fill_grads(wl, 0, scale, g)
            torch.cuda.synchronize()
            opts.append(OneBitAdam(wl.numels, wl.W, params=params, stream=st, **WL.HYPER))
            grads.append(g)
        for o, g in zip(opts, grads):
            o.warmup_step(g)
            o.freeze()
        for _ in range(4):
            if concurrent:
                for o, g in zip(opts, grads):
                    o.step(g)          # queued on different streams, no sync in between
            else:
                for o, g in zip(opts, grads):
                    o.step(g)
                    torch.cuda.synchronize()
        torch.cuda.synchronize()
        out = [(o.read(B.OB_STATE_P), o.read(B.OB_STATE_BITS_SERVER), o.read(B.OB_STATE_E_WORKER, 1))
               for o in opts]
        for o in opts:
            o.close()
        return out

    for a, b in zip(run(True), run(False)):
        for x, y in zip(a, b):
            assert np.array_equal(x.view(np.uint8), y.view(np.uint8))


def test_graph_mode_matches_direct_launches():
    """Graph mode replays the same five kernels: with gradient buffers that
    alternate between steps, the dense -> lazy momentum switch and a
    learning-rate change, it ends bit-identical to direct launches."""
    wl = small_ragged(W=4, count=50)
    runs = []
    for graph in (False, True):
        pr = Pair(wl)
        other = torch.empty_like(pr.grads)
        for _ in range(2):
            pr.warmup_step()
        pr.freeze()
        pr.gpu.graph(graph)
        for k in range(6):
            pr.next_grads()
            g = pr.grads if k % 2 == 0 else other.copy_(pr.grads)
            if k == 3:
                pr.gpu.set_lr(3e-4)
            pr.gpu.step(g)
        runs.append([pr.gpu.read(kd) for kd in (B.OB_STATE_P, B.OB_STATE_M, B.OB_STATE_E_SERVER,
                                                B.OB_STATE_BITS_SERVER, B.OB_STATE_S_WORKER)]
                    + [pr.gpu.read(B.OB_STATE_E_WORKER, w) for w in range(wl.W)])
        pr.close()
    for a, b in zip(*runs):
        assert np.array_equal(a.view(np.uint8), b.view(np.uint8))


def test_steps_captured_by_the_caller_replay_like_direct_launches():
    """With graph mode on (the default) a step queued while the caller
    captures the context's stream is launched kernel by kernel into the
    caller's graph; replaying that graph takes the same steps as direct
    launches, bit for bit."""
    wl = small_ragged(W=4, count=20)
    offs, n_pad = B.ob_layout(wl.numels)
    params = WL.make_params(wl, offs, n_pad, device="cuda")
    scale = WL.grad_scale_vector(wl, offs, n_pad, device="cuda")
    g = torch.empty((wl.W, n_pad), device="cuda")
    s = torch.cuda.Stream()
    cap = OneBitAdam(wl.numels, wl.W, params=params.clone(), stream=s, **WL.HYPER)
    ref = OneBitAdam(wl.numels, wl.W, params=params.clone(), **WL.HYPER)
    ref.graph(False)
    try:
        WL.fill_grads(wl, 0, scale, g)
        torch.cuda.synchronize()
        for o in (cap, ref):
            o.warmup_step(g)
            o.freeze()
        torch.cuda.synchronize()
        WL.fill_grads(wl, 1, scale, g)
        torch.cuda.synchronize()
        for o in (cap, ref):  # the first compressed step reads m densely, later ones lazily
            o.step(g)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            cap.step(g)
        for _ in range(3):
            graph.replay()
            ref.step(g)
        torch.cuda.synchronize()
        for kind in (B.OB_STATE_P, B.OB_STATE_BITS_SERVER, B.OB_STATE_S_SERVER, B.OB_STATE_S_WORKER):
            assert np.array_equal(cap.read(kind).view(np.uint8), ref.read(kind).view(np.uint8)), kind
    finally:
        cap.close()
        ref.close()


def test_set_lr_rejects_non_finite():
    opt = OneBitAdam([100], 2, **WL.HYPER)
    with pytest.raises(B.OnebitError) as ei:
        opt.set_lr(float("nan"))
    assert ei.value.status == B.OB_ERR_INVALID_ARG
    opt.close()
