"""The oracle's multi-tensor runner: with threads > 1 it runs every
(tensor, worker) worker stage and every (tensor, server chunk) server
stage and update as separate jobs; the result must be the sequential
run's bit for bit (the chunks own disjoint elements, words and scales)."""
import numpy as np
import pytest

import oracle

HP = dict(beta1=0.9, beta2=0.999, eps=1e-8, lr=1e-4)


@pytest.mark.parametrize("lamb", [False, True], ids=["adam", "lamb"])
@pytest.mark.parametrize("sizes,W", [((5_001, 777, 0, 40_000, 33), 3), ((100_000, 100, 5), 8),
                                     ((64, 31), 16)])
def test_threaded_runner_equals_sequential(sizes, W, lamb):
    rng = np.random.default_rng(W + len(sizes))
    params = [rng.normal(0, 0.02, n).astype(np.float32) for n in sizes]
    runs = [oracle.OracleRun(params, W, HP, threads=1, lamb=lamb),
            oracle.OracleRun(params, W, HP, threads=4, lamb=lamb)]
    for k in range(5):
        g = [[rng.normal(0, 1e-3, n).astype(np.float32) for n in sizes] for _ in range(W)]
        for r in runs:
            if k < 2:
                r.warmup_step(g)
            else:
                if k == 2:
                    r.freeze()
                r.compressed_step(g)
    a, b = runs
    for t in range(len(sizes)):
        for name in ("p", "m", "e_s", "sbits"):
            np.testing.assert_array_equal(getattr(a, name)[t], getattr(b, name)[t], err_msg=name)
        for w in range(W):
            np.testing.assert_array_equal(a.e_w[w][t], b.e_w[w][t])
            np.testing.assert_array_equal(a.bits_w[w][t], b.bits_w[w][t])
    np.testing.assert_array_equal(a.s_srv, b.s_srv)
    np.testing.assert_array_equal(a.s_w, b.s_w)
    if lamb:
        np.testing.assert_array_equal(a.ratio, b.ratio)
        assert np.all(a.ratio[[t for t, n in enumerate(sizes) if n]] != 1.0)


def test_lamb_runner_with_unit_ratios_is_the_adam_runner():
    """A LAMB run whose every trust ratio is 1 (parameters kept at 0 by a
    learning rate of 0) takes the 1-bit Adam run's steps bit for bit."""
    sizes, W = (3_000, 70, 0), 4
    rng = np.random.default_rng(3)
    hp = dict(HP, lr=0.0)
    params = [np.zeros(n, np.float32) for n in sizes]
    a = oracle.OracleRun(params, W, hp)
    b = oracle.OracleRun(params, W, hp, lamb=True)
    for k in range(5):
        g = [[rng.normal(0, 1e-3, n).astype(np.float32) for n in sizes] for _ in range(W)]
        for r in (a, b):
            if k < 2:
                r.warmup_step(g)
            else:
                if k == 2:
                    r.freeze()
                r.compressed_step(g)
        assert np.all(b.ratio == 1.0)
    for t in range(len(sizes)):
        for name in ("p", "m", "v", "e_s", "sbits"):
            np.testing.assert_array_equal(getattr(a, name)[t], getattr(b, name)[t], err_msg=name)


def _same_state(a, b, sizes, W):
    for t in range(len(sizes)):
        for name in ("p", "m", "e_s", "sbits"):
            np.testing.assert_array_equal(getattr(a, name)[t], getattr(b, name)[t], err_msg=name)
        for w in range(W):
            np.testing.assert_array_equal(a.e_w[w][t], b.e_w[w][t])
            np.testing.assert_array_equal(a.bits_w[w][t], b.bits_w[w][t])
    np.testing.assert_array_equal(a.s_srv, b.s_srv)
    np.testing.assert_array_equal(a.s_w, b.s_w)


@pytest.mark.parametrize("lamb", [False, True], ids=["adam", "lamb"])
@pytest.mark.parametrize("threads", [1, 3])
def test_compressed_step_in_worker_groups_equals_one_call(lamb, threads):
    """The compressed step driven in phases -- the worker stages of groups
    of workers, in any order, then the server stage and update -- is the
    one-call step bit for bit (the form the full-size GPU tests use when
    every worker's gradient does not fit on the host at once)."""
    sizes, W = (5_001, 0, 777, 40_000), 5
    rng = np.random.default_rng(41)
    params = [rng.normal(0, 0.02, n).astype(np.float32) for n in sizes]
    a = oracle.OracleRun(params, W, HP, threads=threads, lamb=lamb)
    b = oracle.OracleRun(params, W, HP, threads=threads, lamb=lamb)
    for k in range(5):
        g = [[rng.normal(0, 1e-3, n).astype(np.float32) for n in sizes] for _ in range(W)]
        if k < 2:
            a.warmup_step(g)
            b.warmup_step(g)
            continue
        if k == 2:
            a.freeze()
            b.freeze()
        a.compressed_step(g)
        b.begin_compressed_step()
        for group in ((3, 1), (4,), (0, 2)):
            b.worker_stages(lambda w: g[w], group)
        b.end_compressed_step()
        _same_state(a, b, sizes, W)
    with pytest.raises(AssertionError):   # a worker left out
        b.begin_compressed_step()
        b.worker_stages(lambda w: g[w], (0, 1, 2, 3))
        b.end_compressed_step()


def test_warmup_reads_gradients_through_device_slices():
    """The warmup fed through gpu_harness.DeviceSlices (slices copied from a
    torch buffer on demand; a CPU tensor here) is the warmup fed numpy
    arrays, bit for bit, threaded or not."""
    torch = pytest.importorskip("torch")
    from gpu_harness import DeviceSlices

    sizes, W = (9_000, 0, 130), 3
    offsets, pos = [], 0
    for n in sizes:
        offsets.append(pos)
        pos += (n + 127) // 128 * 128
    rng = np.random.default_rng(43)
    params = [rng.normal(0, 0.02, n).astype(np.float32) for n in sizes]
    for threads in (1, 4):
        a = oracle.OracleRun(params, W, HP, threads=threads)
        b = oracle.OracleRun(params, W, HP, threads=threads)
        b.SLICE = 1000           # many slices per tensor
        for _ in range(3):
            buf = torch.from_numpy(rng.normal(0, 1e-3, (W, pos)).astype(np.float32))
            host = buf.numpy()
            a.warmup_step([[host[w, o:o + n] for o, n in zip(offsets, sizes)] for w in range(W)])
            b.warmup_step([[DeviceSlices(buf[w], o, n) for o, n in zip(offsets, sizes)]
                           for w in range(W)])
        for t in range(len(sizes)):
            for name in ("p", "m", "v"):
                np.testing.assert_array_equal(getattr(a, name)[t], getattr(b, name)[t])
        full = np.asarray(DeviceSlices(buf[1], offsets[0], sizes[0]))
        np.testing.assert_array_equal(full, buf[1, :sizes[0]].numpy())
