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
