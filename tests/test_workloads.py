"""The synthetic input recipe (seeded generators shared by the CUDA path
and the oracle), on the CPU: the workloads' shapes and sizes, the sweep
grid, and the generators' determinism, zeros, scaling and statistics."""
import math

import numpy as np
import torch

from error_compensated_bit_adam_b200 import _binding as B
from error_compensated_bit_adam_b200 import workloads as WL


def test_workload_sizes():
    assert WL.FLAT_1M_W4.n == 1 << 20 and WL.FLAT_1M_W4.W == 4
    assert WL.BERT_LARGE_FLAT_W8.n == 335_544_320 and WL.BERT_LARGE_FLAT_W8.W == 8
    enc = WL.ENCODER_24L_W16
    assert enc.n_tensors == 338 and enc.n == 333_965_312 and enc.W == 16
    rag = WL.RAGGED_2000_W8
    sizes = [s[0] for s in rag.shapes]
    assert rag.n_tensors == 2000 and rag.n == 519_111_720
    assert min(sizes) >= 1 and max(sizes) <= 1 << 22
    assert sum(n % 32 != 0 for n in sizes) > 1500          # most sizes leave a ragged last word
    grid = {(w.n, w.W) for w in WL.sweep()}
    assert len(grid) == 15 and (1 << 29, 64) not in grid    # 8 W n > 150 GB is skipped


def test_gradient_std_per_tensor():
    enc = WL.ENCODER_24L_W16
    for shape, std in zip(enc.shapes, enc.grad_stds()):
        want = WL.GRAD_STD / math.sqrt(shape[1]) if len(shape) == 2 else WL.GRAD_STD
        assert std == want
    assert WL.FLAT_1M_W4.grad_stds() == [WL.GRAD_STD]


def _small_ragged():
    return WL.Workload("ragged-cpu", WL.ragged_sizes(40, seed=5, max_log2=14), 3, 1, 1, seed=5,
                       zero_fraction=WL.ZERO_FRACTION)


def test_generators_are_deterministic_and_zero_where_promised():
    wl = _small_ragged()
    offsets, n_pad = B.ob_layout(wl.numels)
    scale = WL.grad_scale_vector(wl, offsets, n_pad)
    assert torch.equal(scale, WL.grad_scale_vector(wl, offsets, n_pad))
    p = WL.make_params(wl, offsets, n_pad)
    assert torch.equal(p, WL.make_params(wl, offsets, n_pad))
    real = torch.zeros(n_pad, dtype=torch.bool)
    for o, n in zip(offsets, wl.numels):
        real[o:o + n] = True
    assert (p[~real] == 0).all() and (scale[~real] == 0).all()   # padding
    dropped = real & (scale == 0)
    frac = dropped.sum().item() / real.sum().item()
    assert abs(frac - WL.ZERO_FRACTION) < 0.03                     # the fixed Bernoulli set
    a = torch.empty((wl.W, n_pad))
    b = torch.empty((wl.W, n_pad))
    for step in (0, 7):
        WL.fill_grads(wl, step, scale, a)
        WL.fill_grads(wl, step, scale, b)
        assert torch.equal(a, b)
        zero = a[:, scale == 0]
        assert (zero == 0).all() and not torch.signbit(zero).any()  # exactly +0.0, every worker
    WL.fill_grads(wl, 1, scale, b)
    assert not torch.equal(a, b)                                   # a new draw per step


def test_gradient_statistics():
    wl = WL.flat(1 << 20, 4, seed=9)
    offsets, n_pad = B.ob_layout(wl.numels)
    scale = WL.grad_scale_vector(wl, offsets, n_pad)
    g = torch.empty((wl.W, n_pad))
    WL.fill_grads(wl, 3, scale, g)
    x = g.double().numpy()
    std = WL.GRAD_STD * math.sqrt(2.0)              # shared draw + the worker's own, each N(0, std_t)
    assert abs(x.std() / std - 1) < 0.01 and abs(x.mean()) < 1e-3 * std
    corr = np.corrcoef(x[0], x[1])[0, 1]
    assert abs(corr - 0.5) < 0.01                    # the shared half
    p = WL.make_params(wl, offsets, n_pad).double().numpy()
    assert abs(p.std() / WL.PARAM_STD - 1) < 0.01
