"""Synthetic ablation: 1-bit Adam against error-compensated 1-bit compression
of Adam's gradient, on a noisy, ill-conditioned quadratic.

The review page "1-bit Adam: Communication Efficient Large-Scale Training
with Adam's Convergence Speed" ("Key results", last bullet) reports that
compressing Adam's *gradient* to 1 bit with error compensation does not
give Adam's convergence, which is why 1-bit Adam freezes the variance after
a warmup and compresses the momentum instead.  This experiment checks that
claim on a problem with no dataset:

    f(p) = mean_i h_i (p_i - p*_i)^2 / 2,   h_i log-uniform in [h_min, h_max],

with W workers whose gradients are h (p - p*) plus independent Gaussian
noise.  Three arms start from the same p0 and take the same gradients:

  adam       full-precision Adam on the averaged gradient every step (the
             library's warmup step, never frozen);
  onebit     1-bit Adam: the same Adam for the first `warmup` steps, then
             the freeze and the library's compressed steps;
  ec_grad    the same Adam warmup, then Adam (moments continued from the
             warmup's) driven by the gradient after the library's
             error-compensated 1-bit compressed allreduce (a context with
             beta1 = 0, whose worker stage then compresses g_w + e_w, and lr
             = 0, so its decoded momentum is the compressed average
             gradient); the Adam update itself is a few torch operations.

Every step of both 1-bit arms runs the library's kernels.  The result is
reported as it comes out, whatever it shows.

    python -m error_compensated_bit_adam_b200.ablation [--n N] [--workers W]
        [--steps T] [--warmup Tw] [--noise SIGMA ...] [--lr LR ...] [--h-min H ...] [--seed S]
"""
from __future__ import annotations

import argparse
import json
import math
import time
from typing import Dict, List

import torch

from . import _binding as B
from .optimizer import OneBitAdam


def make_problem(n: int, seed: int, h_min: float, h_max: float, dev):
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    u = torch.rand(n, generator=g, device=dev, dtype=torch.float64)
    h = torch.exp(math.log(h_min) + u * (math.log(h_max) - math.log(h_min)))
    p_star = torch.randn(n, generator=g, device=dev, dtype=torch.float64)
    p0 = torch.randn(n, generator=g, device=dev, dtype=torch.float64)
    return h, p_star, p0


def loss(p: torch.Tensor, h: torch.Tensor, p_star: torch.Tensor) -> float:
    d = p.double() - p_star
    return float(0.5 * torch.mean(h * d * d))


def gradients(p, h, p_star, W, noise, gen, out):
    """out[w] = h (p - p*) + noise * N(0, 1), fp32."""
    clean = (h * (p.double() - p_star)).float()
    out.normal_(0.0, noise, generator=gen)
    out += clean


def run(n: int = 1 << 20, W: int = 8, steps: int = 2000, warmup: int = 400, noise: float = 0.1,
        lr: float = 1e-2, seed: int = 7, h_min: float = 1e-3, h_max: float = 10.0,
        every: int = 50, device="cuda") -> Dict[str, List[float]]:
    dev = torch.device(device)
    h, p_star, p0 = make_problem(n, seed, h_min, h_max, dev)
    hyper = dict(beta1=0.9, beta2=0.999, eps=1e-8, lr=lr)
    curves: Dict[str, List[float]] = {}
    for arm in ("adam", "onebit", "ec_grad"):
        gen = torch.Generator(device=dev)
        gen.manual_seed(seed + 1)                      # the same gradient noise in every arm
        opt = OneBitAdam([n], W, params=p0.float().clone(), device=dev, **hyper)
        comp = None
        g = torch.empty((W, opt.n_padded), dtype=torch.float32, device=dev)
        g.zero_()
        rows = g[:, :n]
        curve = [loss(opt.params[:n], h, p_star)]
        m = v = None
        for t in range(1, steps + 1):
            gradients(opt.params[:n], h, p_star, W, noise, gen, rows)
            if arm == "adam" or t <= warmup:
                opt.warmup_step(g)
            elif arm == "onebit":
                if t == warmup + 1:
                    opt.freeze()
                opt.step(g)
            else:
                if comp is None:                       # Adam's state after the warmup
                    m = torch.from_numpy(opt.read(B.OB_STATE_M)).to(dev)
                    v = torch.from_numpy(opt.read(B.OB_STATE_V)).to(dev)
                    comp = OneBitAdam([n], W, device=dev, beta1=0.0, beta2=0.999, eps=1e-8, lr=0.0)
                    comp.warmup_step(torch.zeros_like(g))
                    comp.freeze()
                comp.step(g)                           # error-compensated 1-bit allreduce of g
                gh = torch.from_numpy(comp.read(B.OB_STATE_M)).to(dev)
                m.mul_(hyper["beta1"]).add_(gh, alpha=1 - hyper["beta1"])
                v.mul_(hyper["beta2"]).addcmul_(gh, gh, value=1 - hyper["beta2"])
                bc1 = 1 - hyper["beta1"] ** t
                bc2 = 1 - hyper["beta2"] ** t
                opt.params.sub_(lr * (m / bc1) / ((v / bc2).sqrt() + hyper["eps"]))
            if t % every == 0:
                curve.append(loss(opt.params[:n], h, p_star))
        torch.cuda.synchronize(dev)
        curves[arm] = curve
        opt.close()
        if comp is not None:
            comp.close()
    return curves


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--n", type=int, default=1 << 20)
    ap.add_argument("--workers", type=int, default=8)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=400)
    ap.add_argument("--noise", type=float, nargs="+", default=[0.01, 0.1, 1.0])
    ap.add_argument("--lr", type=float, nargs="+", default=[1e-2, 1e-3])
    ap.add_argument("--h-min", type=float, nargs="+", default=[1e-3, 1e-1],
                    help="smallest curvature (the largest is --h-max): 1e-3 is ill-conditioned")
    ap.add_argument("--h-max", type=float, default=10.0)
    ap.add_argument("--every", type=int, default=50)
    ap.add_argument("--seed", type=int, default=7)
    args = ap.parse_args(argv)
    for h_min in args.h_min:
        for lr in args.lr:
            for noise in args.noise:
                t0 = time.time()
                curves = run(args.n, args.workers, args.steps, args.warmup, noise, lr, args.seed,
                             h_min=h_min, h_max=args.h_max, every=args.every)
                print(json.dumps({"n": args.n, "W": args.workers, "steps": args.steps,
                                  "warmup": args.warmup, "noise": noise, "lr": lr, "h_min": h_min,
                                  "h_max": args.h_max, "seed": args.seed, "every": args.every,
                                  "seconds": time.time() - t0, "loss": curves}), flush=True)


if __name__ == "__main__":
    main()
