"""Seeded synthetic workloads for the compression-phase step of 1-bit Adam.

This module holds only input generation: tensor shapes, hyperparameters and
seeded random parameters / gradients.  It contains none of the method's
arithmetic, and it is the one module that both the product path's
callers (tests, benchmark) and the oracle's callers share.

The workloads stand in for the BERT-Large training runs on the review page
"1-bit Adam: Communication Efficient Large-Scale Training with Adam's
Convergence Speed" (section "Key results"): no dataset or checkpoint is
used.  Recipe, for every workload:

* parameters ~ N(0, 0.02);
* per step k and worker w: g_w = g_shared + noise_w, both ~ N(0, std_t),
  with std_t = 1e-3 (flat vectors, 1-D tensors) or 1e-3/sqrt(fan_in) for a
  2-D tensor of shape (out, in), fan_in = in;
* the ragged workload zeroes a fixed Bernoulli(0.2) subset of the gradient
  entries (the same subset for every worker and step);
* hyperparameters beta1 = 0.9, beta2 = 0.999, eps = 1e-8, lr = 1e-4.

Gradients are written into a flat buffer laid out by caller-supplied tensor
offsets (padding entries are 0).  Random numbers come from torch generators
seeded by (workload seed, step, stream); CPU and CUDA generators give
different but individually reproducible streams.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import numpy as np
import torch

HYPER = dict(beta1=0.9, beta2=0.999, eps=1e-8, lr=1e-4)

PARAM_STD = 0.02
GRAD_STD = 1e-3
ZERO_FRACTION = 0.2


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    shapes: tuple            # per-tensor shapes
    W: int                   # simulated data-parallel workers
    warmup_steps: int        # full-precision Adam steps before the freeze
    compressed_steps: int    # compression-phase steps
    seed: int
    fan_in_scaling: bool = False
    zero_fraction: float = 0.0

    @property
    def numels(self) -> List[int]:
        return [int(np.prod(s)) if len(s) else 1 for s in self.shapes]

    @property
    def n(self) -> int:
        return sum(self.numels)

    @property
    def n_tensors(self) -> int:
        return len(self.shapes)

    def grad_stds(self) -> List[float]:
        out = []
        for s in self.shapes:
            if self.fan_in_scaling and len(s) == 2:
                out.append(GRAD_STD / math.sqrt(s[1]))
            else:
                out.append(GRAD_STD)
        return out

    def describe(self) -> str:
        return (f"{self.name}: {self.n_tensors} fp32 tensor(s), n={self.n}, W={self.W}, "
                f"{self.warmup_steps} Adam warmup + {self.compressed_steps} compressed steps")


def encoder_shapes(layers: int = 24, hidden: int = 1024, ffn: int = 4096, vocab: int = 30522,
                   positions: int = 512) -> tuple:
    """Per layer: four hidden x hidden matrices, one hidden x ffn, one
    ffn x hidden and eight hidden-long bias/norm vectors; then a vocab x
    hidden and a positions x hidden embedding."""
    per_layer = ([(hidden, hidden)] * 4 + [(hidden, ffn), (ffn, hidden)] + [(hidden,)] * 8)
    return tuple(per_layer * layers + [(vocab, hidden), (positions, hidden)])


def ragged_sizes(count: int, seed: int, max_log2: int = 22) -> tuple:
    """count sizes max(1, floor(2^(max_log2 * u))), u ~ U[0, 1) from seed."""
    u = np.random.default_rng(seed).random(count)
    return tuple((max(1, int(math.floor(2.0 ** (max_log2 * x)))),) for x in u)


def flat(n: int, W: int, warmup: int = 5, compressed: int = 10, seed: int = 50,
         name: Optional[str] = None) -> Workload:
    return Workload(name or f"flat-n{n}-W{W}", ((n,),), W, warmup, compressed, seed)


# The five workloads of the benchmark suite.
FLAT_1M_W4 = Workload("flat-1M-W4", ((1 << 20,),), 4, 5, 10, seed=11)
BERT_LARGE_FLAT_W8 = Workload("bert-large-flat-336M-W8", ((335_544_320,),), 8, 100, 50, seed=12)
ENCODER_24L_W16 = Workload("encoder-24L-h1024-ffn4096-W16", encoder_shapes(), 16, 5, 10, seed=13,
                           fan_in_scaling=True)
RAGGED_2000_W8 = Workload("ragged-2000-W8", ragged_sizes(2000, seed=14), 8, 5, 10, seed=14,
                          zero_fraction=ZERO_FRACTION)
SWEEP_N = (1 << 20, 1 << 24, 1 << 27, 1 << 29)
SWEEP_W = (2, 8, 32, 64)
SWEEP_STATE_LIMIT_BYTES = 150e9


def sweep() -> List[Workload]:
    """n x W grid, skipping points whose per-worker state (8 bytes per
    parameter per worker: gradient + error) exceeds 150 GB."""
    out = []
    for n in SWEEP_N:
        for W in SWEEP_W:
            if 8.0 * W * n > SWEEP_STATE_LIMIT_BYTES:
                continue
            out.append(flat(n, W, seed=15, name=f"sweep-n{n}-W{W}"))
    return out


WORKLOADS = {w.name: w for w in (FLAT_1M_W4, BERT_LARGE_FLAT_W8, ENCODER_24L_W16, RAGGED_2000_W8)}


# ---------------------------------------------------------------------------
# seeded generation
# ---------------------------------------------------------------------------

def _mix(*parts: int) -> int:
    h = 0x9E3779B97F4A7C15
    for p in parts:
        h ^= (int(p) + 0x9E3779B97F4A7C15 + ((h << 6) & 0xFFFFFFFFFFFFFFFF) + (h >> 2))
        h &= 0xFFFFFFFFFFFFFFFF
    return h & 0x7FFFFFFFFFFFFFFF


def _gen(device, *parts: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_mix(*parts))
    return g


def dense_offsets(numels: Sequence[int]) -> List[int]:
    """Back-to-back offsets (no padding), for callers that need none."""
    out, acc = [], 0
    for n in numels:
        out.append(acc)
        acc += n
    return out


def grad_scale_vector(wl: Workload, offsets: Sequence[int], total: int,
                      device="cpu") -> torch.Tensor:
    """float32[total]: the gradient std of each entry; 0 on padding and on
    the ragged workload's zeroed subset."""
    scale = torch.zeros(total, dtype=torch.float32, device=device)
    for t, (off, n, std) in enumerate(zip(offsets, wl.numels, wl.grad_stds())):
        scale[off:off + n] = std
    if wl.zero_fraction > 0:
        g = _gen(device, wl.seed, 0x2E20)
        drop = torch.rand(total, generator=g, device=device) < wl.zero_fraction
        scale[drop] = 0.0
    return scale


def make_params(wl: Workload, offsets: Sequence[int], total: int, device="cpu") -> torch.Tensor:
    """float32[total]: parameters ~ N(0, 0.02), padding 0."""
    g = _gen(device, wl.seed, 0x9A7A)
    raw = torch.randn(total, generator=g, device=device, dtype=torch.float32) * PARAM_STD
    out = torch.zeros(total, dtype=torch.float32, device=device)
    for off, n in zip(offsets, wl.numels):
        out[off:off + n] = raw[off:off + n]
    return out


def fill_grads(wl: Workload, step: int, scale: torch.Tensor, out: torch.Tensor) -> None:
    """out[w, :] = (z_shared + z_w) * scale for step `step` (0-based over the
    whole run, warmup and compressed steps counted together)."""
    W, total = out.shape
    assert W == wl.W and scale.numel() == total
    dev = out.device
    z_shared = torch.randn(total, generator=_gen(dev, wl.seed, step, 1 << 20), device=dev,
                           dtype=torch.float32)
    shared = z_shared * scale
    del z_shared
    zero = scale == 0  # padding and zeroed entries: make them exactly +0.0
    any_zero = bool(zero.any())
    for w in range(W):
        z = torch.randn(total, generator=_gen(dev, wl.seed, step, w), device=dev,
                        dtype=torch.float32)
        torch.mul(z, scale, out=out[w])
        out[w].add_(shared)
        if any_zero:
            out[w].masked_fill_(zero, 0.0)


def split(flat_buf: np.ndarray, offsets: Sequence[int], numels: Sequence[int]) -> List[np.ndarray]:
    """Per-tensor dense copies out of a flat laid-out numpy buffer."""
    return [np.ascontiguousarray(flat_buf[o:o + n]) for o, n in zip(offsets, numels)]
