#!/usr/bin/env python
"""Benchmark of the compression-phase step of 1-bit Adam on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]
                    [--workload NAME | --n N --workers W] [--adam-steps S]

One step = one ob_compressed_step over the whole workload: worker stage
(momentum, error feedback, 1-bit compression) for every simulated worker,
server stage, gather and preconditioned update.  Default workload: the
BERT-Large-sized flat fp32 vector, n = 335,544,320, W = 8 simulated
workers, after 100 full-precision Adam warmup steps and the freeze.

Prints one JSON line (rank 0).  value = parameters updated per second per
worker.  With one GPU all W workers are simulated in its HBM and the
exchange is addressing inside it.  With N > 1 GPUs (torchrun, one process
per GPU) the W workers are spread over the GPUs, W/N each, and every step
runs the split step with its per-chunk NCCL exchange between them (value =
n / the slowest rank's step time, "strong" scaling); --multi replicas runs
N independent one-GPU steps instead ("weak").

--impl reference times the CPU oracle (single-threaded C) on a bounded
sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from error_compensated_bit_adam_b200 import _binding as B  # noqa: E402
from error_compensated_bit_adam_b200 import workloads as WL  # noqa: E402

METRIC = "params updated/s per virtual worker (W=8, 336M fp32) and HBM GB/s as % of peak"
UNIT = "params/s per virtual worker"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0
GRAD_SETS = 2


# ----------------------------------------------------------------- helpers

def algorithmic_bytes(n_real: int, W: int, lamb: bool = False) -> dict:
    """Bytes each kernel of a steady-state compressed step must move, per
    real parameter, in this formulation (errors stored as (x, s) and the
    momentum as last step's server words and scales):
      pack    1/8 (server words -> m) + W (4 g + 4 x_prev + 4 x) + W/8 (words)
      server  W/8 (words) + 4 (y_prev) + 4 (y) + 1/8 (words)
      apply   1/8 (words) + 4 (d) + 8 (p read and write)   (1-bit LAMB's
              update the same, plus per-tile sums of ~0)
      warmup  4W (g) + 24 (m, v, p read and write)   [pre-path]
              1-bit LAMB: 4W + 20 (moments: g, m, v, p read; m, v
              written) + 16 (step: m, v, p read; p written)
      freeze  8 (v read, d written)                  [pre-path]
    The scale kernels move ~0.  'model' is the dense-momentum byte model
    12W + W/4 + 28.25 (126.25 B at W=8) the effective-bandwidth target is
    quoted on."""
    pack = n_real * (1 / 8 + 12 * W + W / 8)
    server = n_real * (W / 8 + 8 + 1 / 8)
    apply = n_real * (1 / 8 + 4 + 8)
    return {"ob_pack_kernel": pack, "ob_server_kernel": server, "ob_apply_kernel": apply,
            "step": pack + server + apply, "model": n_real * (12 * W + W / 4 + 28.25),
            # the untimed pre-path: Adam reads W gradients and reads and
            # writes m, v and p; the freeze reads v and writes d in its place
            "ob_warmup_kernel": n_real * (4 * W + (36 if lamb else 24)), "ob_freeze_kernel": n_real * 8}


# With 1-bit LAMB the warmup and update slots of the profiling counters time
# LAMB's kernels: their DRAM traffic is looked up under LAMB's own entries.
LAMB_TRAFFIC_KEYS = {"ob_warmup_kernel": "ob_lamb_warmup", "ob_apply_kernel": "ob_lamb_apply_kernel"}


def traffic_key(name: str, lamb: bool) -> str:
    return LAMB_TRAFFIC_KEYS.get(name, name) if lamb else name


def kernel_sources_sha256(files) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "error_compensated_bit_adam_b200", "csrc", "kernels", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(kernel: str, n: int, W: int):
    """DRAM bytes per launch of `kernel` from the ncu capture recorded in
    profiles/ncu_traffic.json, scaled to n parameters; None when no capture
    exists for this W or the kernel's sources changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        entry = rec["kernels"][kernel]
        if entry["W"] != W or kernel_sources_sha256(entry["sources"]) != entry["sources_sha256"]:
            return None
        return entry["dram_bytes_per_param"] * n
    except Exception:
        return None


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled while timing.

    start() launches the sampler and waits for its first sample (nvidia-smi
    needs about a second to start); mark() and stop() bracket the timed
    region, and only the samples stamped inside it are reported (or, for a
    region shorter than one interval, the sample nearest its end)."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    N_FIELDS = 10

    def __init__(self, interval_ms=50):
        self.proc = None
        self.path = None
        self.interval_ms = interval_ms
        self.t_start = None

    def _rows(self):
        import datetime
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) != self.N_FIELDS:
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                except ValueError:
                    continue
                rows.append((ts, parts[1:]))
        return rows

    def start(self, ready_timeout_s=5.0):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 f"-lms", str(self.interval_ms)], stdout=self.out, stderr=subprocess.DEVNULL)
            t_end = time.time() + ready_timeout_s
            while time.time() < t_end and self.proc.poll() is None and not self._rows():
                time.sleep(0.02)
        except Exception:
            self.proc = None

    def mark(self):
        self.t_start = time.time()

    def stop(self):
        if self.proc is None:
            return None
        t_stop = time.time()
        time.sleep(2 * self.interval_ms / 1000.0)  # the sample that covers the region's end
        try:
            self.proc.terminate()
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        rows = self._rows()
        os.unlink(self.path)
        t_start = self.t_start if self.t_start is not None else t_stop
        inside = [r for ts, r in rows if t_start <= ts <= t_stop]
        if not inside:
            before = [r for ts, r in rows if ts <= t_stop]
            inside = before[-1:] or [r for _, r in rows][:1]
        if not inside:
            return None
        sm = [float(r[1]) for r in inside if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in inside if r[2].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in inside:
            for name, val in zip(names, r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(inside)}


def pick_workload(args) -> WL.Workload:
    if args.n:
        return WL.flat(args.n, args.workers, warmup=args.adam_steps or 2, compressed=0, seed=31,
                       name=f"flat-n{args.n}-W{args.workers}")
    names = dict(WL.WORKLOADS)
    for w in WL.sweep():
        names[w.name] = w
    wl = names[args.workload]
    if args.adam_steps is not None:
        wl = WL.Workload(wl.name, wl.shapes, wl.W, args.adam_steps, wl.compressed_steps, wl.seed,
                         wl.fan_in_scaling, wl.zero_fraction)
    return wl


def workload_config(wl: WL.Workload, n_pad: int, parallelism: str, grad_sets: int = GRAD_SETS) -> dict:
    return {"workload": wl.describe(), "n": wl.n, "n_padded": n_pad, "W": wl.W,
            "tensors": wl.n_tensors, "adam_warmup_steps": wl.warmup_steps,
            "grad_sets_cycled": grad_sets,
            "l2": f"inputs larger than L2: {4 * wl.W * n_pad / 1e9:.2f} GB of gradients per step",
            "parallelism": parallelism}


# ------------------------------------------------------------ oracle timing

ORACLE_SAMPLE = 1 << 21  # elements of the flat vector the oracle is timed on (both legs)


def oracle_sample_rate(W: int, n_sample: int, steps: int, warm: int = 1, threads: int = 1):
    """Time the oracle's compressed step (single-threaded C calls; with
    threads > 1 its independent per-worker and per-chunk calls run
    concurrently) on a flat n_sample vector with W workers; returns
    (params/s per worker, seconds per step).  Inputs come from the shared
    generator, on the CPU."""
    import oracle
    wl = WL.flat(n_sample, W, warmup=1, compressed=steps, seed=41, name="oracle-sample")
    offs = [0]
    p = WL.make_params(wl, offs, n_sample).numpy()
    scale = WL.grad_scale_vector(wl, offs, n_sample)
    run = oracle.OracleRun([p], W, WL.HYPER, threads=threads)
    g = torch.empty((W, n_sample), dtype=torch.float32)
    WL.fill_grads(wl, 0, scale, g)
    run.warmup_step([[g[w].numpy()] for w in range(W)])
    run.freeze()
    times = []
    for k in range(warm + steps):
        WL.fill_grads(wl, 1 + k, scale, g)
        gl = [[g[w].numpy()] for w in range(W)]
        t0 = time.perf_counter()
        run.compressed_step(gl)
        dt = time.perf_counter() - t0
        if k >= warm:
            times.append(dt)
    t = sum(times) / len(times)
    return n_sample / t, t


def cpu_baseline(W: int, n_sample: int = ORACLE_SAMPLE, steps: int = 8) -> dict:
    rate, t = oracle_sample_rate(W, n_sample, steps)
    out = {"value": rate, "unit": UNIT, "cores": 1, "kind": "oracle",
           "sample": f"flat fp32 n={n_sample}, W={W}: {steps} timed oracle compressed steps "
                     f"({t:.2f} s each) after 1 Adam step and the freeze; single-threaded C"}
    cores = os.cpu_count() or 1
    if cores > 1 and W > 1:  # a second, separately labelled figure: the same calls on every core
        threads = min(cores, W)
        trate, tt = oracle_sample_rate(W, n_sample, steps, threads=threads)
        out["threaded"] = {"value": trate, "unit": UNIT, "cores": threads, "kind": "oracle",
                           "sample": f"the same sample, its {W} worker stages and {W} server "
                                     f"chunks run as concurrent single-threaded calls "
                                     f"({tt:.2f} s per step)"}
    return out


# ------------------------------------------------------------- reference arm

def run_reference(args) -> None:
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = pick_workload(args)
    n_sample = min(wl.n, ORACLE_SAMPLE)
    rate, t = oracle_sample_rate(wl.W, n_sample, args.steps, warm=args.warmup)
    line = {
        "impl": "reference", "metric": METRIC, "value": rate, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": workload_config(wl, wl.n, "cpu, single thread"),
        "cpu_baseline": {"value": rate, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"flat fp32 n={n_sample} of the workload's shape, W={wl.W}; "
                                   f"{args.warmup} untimed + {args.steps} timed oracle steps"},
        "e2e": {"value": rate, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------- b200 arm

def max_over_ranks(x: float, world: int) -> float:
    if world <= 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(n_per_replica: int, world: int, ms_per_step_max: float) -> float:
    """Whole-job parameters updated per second per simulated worker: every
    rank updates its own replica of n parameters each step, and the step
    time is the slowest rank's."""
    return world * n_per_replica / (ms_per_step_max / 1e3)


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def measure_e2e(opt, wl, n_pad, dev_grads, args, world, dev) -> dict:
    """The step through the public host-buffer call: every step copies W
    gradient vectors from pinned host memory to the GPU (overlapped with the
    worker stage) and reads the step's server scales back."""
    # Every rank takes the same collective steps whatever happens locally
    # (a failure is carried as a flag), so no rank waits on another.
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    err, pinned, host, out, elapsed = None, False, None, None, 0.0
    try:
        try:
            host = torch.empty((wl.W, n_pad), dtype=torch.float32, pin_memory=True)
            pinned = True
        except RuntimeError:
            host = torch.empty((wl.W, n_pad), dtype=torch.float32)
        host.copy_(dev_grads)
        out = np.zeros(wl.n_tensors * wl.W, np.float32)
        opt.step_host(host, out)                    # untimed: staging allocation
        if torch.cuda.is_available():
            torch.cuda.synchronize(dev)
    except Exception as exc:  # reported, never hidden
        err = repr(exc)
    barrier(world)
    if err is None:
        try:
            w0 = time.perf_counter()
            for _ in range(e2e_steps):
                opt.step_host(host, out)
            elapsed = time.perf_counter() - w0
        except Exception as exc:
            err = repr(exc)
    e2e_s = max_over_ranks(elapsed, world) / e2e_steps
    failed = max_over_ranks(0.0 if err is None else 1.0, world)
    if failed:
        return {"value": None, "unit": UNIT, "error": err or "failed on another rank"}
    return {"value": world * wl.n / e2e_s, "unit": UNIT,
            "h2d_bytes_per_step": int(host.numel() * 4), "d2h_bytes_per_step": int(out.nbytes),
            "ms_per_step": e2e_s * 1e3, "pinned": pinned, "steps": e2e_steps,
            "call": "ob_compressed_step_host"}


def measure_split_ranks(wl, args, dev) -> dict:
    """The split step (distributed.LocalRanks) as G ranks on this one GPU,
    each with its own context, the exchanges done by device copies: each
    rank's own kernels (worker stage of W/G workers, server stage of its
    chunks, the update) timed by its context's event pairs.  That is the
    compute of one GPU in a G-GPU run; the exchange over NVLink is not
    measured here (one GPU), only its bytes are reported."""
    from error_compensated_bit_adam_b200.distributed import LocalRanks
    G = args.split_ranks
    offsets, n_pad = B.ob_layout(wl.numels)
    need = G * (B.ob_workspace_bytes(wl.numels, wl.W) + 4 * n_pad) + 4 * wl.W * n_pad + (1 << 30)
    free = torch.cuda.mem_get_info(dev)[0]
    if free < need:
        return {"G": G, "skipped": f"needs {need / 1e9:.1f} GB of device memory, {free / 1e9:.1f} free"}
    params = WL.make_params(wl, offsets, n_pad, device=dev)
    scale = WL.grad_scale_vector(wl, offsets, n_pad, device=dev)
    ranks = LocalRanks(wl.numels, wl.W, G, device=dev, **WL.HYPER)
    g = torch.empty((wl.W, n_pad), dtype=torch.float32, device=dev)
    try:
        for r in ranks.ranks:
            r.params.copy_(params)
        del params
        WL.fill_grads(wl, 0, scale, g)
        ranks.warmup_step(g)
        ranks.freeze()
        WL.fill_grads(wl, 1, scale, g)
        del scale
        for _ in range(max(1, args.warmup)):
            ranks.step(g)
        torch.cuda.synchronize(dev)
        for r in ranks.ranks:
            r.opt.profile(True)
            r.opt.profile_read(reset=True)
        K = max(1, min(args.steps, 20))
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(K):
            ranks.step(g)
        t1.record()
        torch.cuda.synchronize(dev)
        per_rank = []
        for r in ranks.ranks:
            prof = r.opt.profile_read(reset=True)
            r.opt.profile(False)
            per_rank.append({name: ms / K for name, (ms, cnt) in prof.items() if cnt})
        compute = [sum(p.values()) for p in per_rank]
        return {"G": G, "W": wl.W, "workers_per_rank": wl.W // G, "steps": K,
                "ms_per_step_all_ranks_on_one_gpu": t0.elapsed_time(t1) / K,
                "rank_compute_ms_per_step": compute,
                "rank0_kernels_ms_per_step": per_rank[0],
                "exchange_bytes_per_rank_per_step": ranks.ranks[0].exchange_bytes(),
                "note": "each rank's own kernels, timed by its context; the exchange between "
                        "ranks is device copies on one GPU here, not NVLink, and is not timed"}
    finally:
        ranks.close()


def measure_overlap(wl, args, dev, world) -> dict:
    """Bucketed compressed steps overlapping a synthetic backward pass.

    The tensor list is cut into buckets of about --bucket-elems elements,
    each stepped by its own context on its own stream (graph mode).  The
    backward of bucket b is modelled as two bf16 GEMMs of 2 * tokens * n_b
    FLOPs each (weight and input gradients of n_b parameters over
    --overlap-tokens tokens), run on the main stream in reverse bucket order;
    bucket b's step starts when its backward GEMMs are done.  Reports the
    backward alone, the steps alone, both interleaved, and the share of the
    shorter of the two that the interleaving hid."""
    from error_compensated_bit_adam_b200.buckets import BucketedOneBitAdam, split_buckets
    buckets = split_buckets(wl.numels, args.bucket_elems)
    bk = BucketedOneBitAdam(wl.numels, wl.W, buckets, graph=True, device=dev,
                            priority=args.overlap_priority, **WL.HYPER)
    grads = []
    for b, ts in enumerate(buckets):
        sub = WL.Workload(f"{wl.name}-bucket{b}", tuple(wl.shapes[t] for t in ts), wl.W, 0, 0,
                          wl.seed + 1000 + b, wl.fan_in_scaling, wl.zero_fraction)
        offs, n_pad = bk.layout(b)
        g = torch.empty((wl.W, n_pad), dtype=torch.float32, device=dev)
        WL.fill_grads(sub, 0, WL.grad_scale_vector(sub, offs, n_pad, device=dev), g)
        grads.append(g)
    K = 1024
    gemms = []
    for ts in buckets:
        n_b = sum(wl.numels[t] for t in ts)
        N = max(1, -(-n_b // K))
        a = torch.randn(args.overlap_tokens, K, device=dev, dtype=torch.bfloat16)
        w = torch.randn(K, N, device=dev, dtype=torch.bfloat16)
        gemms.append((a, w, torch.empty(args.overlap_tokens, N, device=dev, dtype=torch.bfloat16),
                      torch.empty(K, N, device=dev, dtype=torch.bfloat16)))

    def backward(b):
        a, w, out_x, out_w = gemms[b]
        torch.matmul(a, w, out=out_x)              # input-gradient-sized GEMM
        torch.matmul(a.t(), out_x, out=out_w)      # weight-gradient-sized GEMM

    torch.cuda.synchronize(dev)
    for b in range(len(buckets)):
        bk.warmup_step(b, grads[b])
    bk.wait()
    bk.freeze()
    for _ in range(2):
        for b in range(len(buckets)):
            bk.step(b, grads[b])
            backward(b)
    bk.wait()
    torch.cuda.synchronize(dev)

    def timed(run, reps):
        barrier(world)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            run()
        e1.record()
        torch.cuda.synchronize(dev)
        return max_over_ranks(e0.elapsed_time(e1), world) / reps

    order = list(reversed(range(len(buckets))))

    def only_backward():
        for b in order:
            backward(b)

    def only_steps():
        for b in order:
            bk.step(b, grads[b])
        bk.wait()

    def both():
        for b in order:
            backward(b)
            ev = torch.cuda.Event()
            ev.record()
            bk.step(b, grads[b], ev)
        bk.wait()

    reps = max(3, min(args.steps, 10))
    t_b, t_s, t_o = timed(only_backward, reps), timed(only_steps, reps), timed(both, reps)
    flops = sum(4 * args.overlap_tokens * K * max(1, -(-sum(wl.numels[t] for t in ts) // K))
                for ts in buckets)
    bk.close()
    return {"buckets": len(buckets), "bucket_elems": args.bucket_elems,
            "stream_priority": args.overlap_priority,
            "backward_model": f"2 bf16 GEMMs per bucket, {args.overlap_tokens} tokens, "
                              f"{flops / 1e12:.2f} TFLOP per pass",
            "backward_ms": t_b, "steps_ms": t_s, "overlapped_ms": t_o,
            "sequential_ms": t_b + t_s,
            "hidden_fraction_of_shorter": (t_b + t_s - t_o) / min(t_b, t_s)}


def run_split(args, world: int, rank: int, dev) -> None:
    """The workload's W workers spread over the `world` processes, one per
    GPU, through the split step (distributed.DistributedOneBitAdam): each
    process runs the worker stage of its W/world workers, exchanges chunks
    of the worker words with the others (NCCL point-to-point), serves its
    share of the server chunks, exchanges the server words and scales, and
    updates.  The whole job updates n parameters per step for each of the
    W workers, so value = n / step time (the slowest rank's), the total
    work fixed as the GPUs grow ("strong")."""
    from error_compensated_bit_adam_b200.distributed import DistributedOneBitAdam

    wl = pick_workload(args)
    if wl.W % world:
        raise SystemExit(f"W = {wl.W} workers do not split over {world} GPUs")
    offsets, n_pad = B.ob_layout(wl.numels)
    params = WL.make_params(wl, offsets, n_pad, device=dev)
    scale = WL.grad_scale_vector(wl, offsets, n_pad, device=dev)
    D = DistributedOneBitAdam(wl.numels, wl.W, rank=rank, world=world, device=dev,
                              peer_words=args.peer_words and world > 1, **WL.HYPER)
    D.params.copy_(params)
    del params
    wl_local, w0 = D.w_local, D.w_begin
    full = torch.empty((wl.W, n_pad), dtype=torch.float32, device=dev)
    step = 0
    D.opt.profile(True)
    for _ in range(wl.warmup_steps):           # Adam on all-reduced gradients, outside the step
        WL.fill_grads(wl, step, scale, full)
        step += 1
        D.warmup_step_allreduce([full[w0 + i] for i in range(wl_local)])
    D.freeze()
    pre_prof = D.opt.profile_read(reset=True)
    D.opt.profile(False)
    grads = []
    for _ in range(GRAD_SETS):                 # this process's workers' rows of fresh draws
        WL.fill_grads(wl, step, scale, full)
        step += 1
        grads.append(full[w0:w0 + wl_local].clone())
    del full, scale
    local_rows = [[g[i] for i in range(wl_local)] for g in grads]
    for k in range(args.warmup):
        D.step(local_rows[k % len(grads)])
    torch.cuda.synchronize(dev)

    stream = D.opt.stream
    D.opt.profile(True)
    D.opt.profile_read(reset=True)
    sampler = ClockSampler()
    if rank == 0:
        sampler.start()
    barrier(world)
    torch.cuda.synchronize(dev)
    sampler.mark()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for k in range(args.steps):
        D.step(local_rows[k % len(grads)])
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    clocks = sampler.stop() if rank == 0 else None
    prof = D.opt.profile_read(reset=True)
    D.opt.profile(False)
    ms_per_step = max_over_ranks(t0.elapsed_time(t1), world) / args.steps
    launches = sum(prof[B.ob_kernel_name(k)][1] for k in range(B.OB_K_PACK, B.OB_K_APPLY + 1))
    launches = int(max_over_ranks(float(launches), world)) * world

    # end to end: every step copies this process's gradients in from pinned
    # host memory and reads the step's server scales back
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    host = [torch.empty((wl_local, n_pad), dtype=torch.float32, pin_memory=True) for _ in range(1)]
    host[0].copy_(grads[0])
    scales_out = torch.empty(D.server_scales.numel(), dtype=torch.float32, pin_memory=True)
    dev_rows = grads[0]
    barrier(world)
    torch.cuda.synchronize(dev)
    w_start = time.perf_counter()
    for _ in range(e2e_steps):
        with torch.cuda.stream(stream):
            dev_rows.copy_(host[0], non_blocking=True)
        D.step(local_rows[0])
        with torch.cuda.stream(stream):
            scales_out.copy_(D.server_scales, non_blocking=True)
        stream.synchronize()
    e2e_s = max_over_ranks(time.perf_counter() - w_start, world) / e2e_steps
    e2e = {"value": wl.n / e2e_s, "unit": UNIT, "h2d_bytes_per_step": int(host[0].numel() * 4 * world),
           "d2h_bytes_per_step": int(scales_out.numel() * 4 * world), "ms_per_step": e2e_s * 1e3,
           "steps": e2e_steps, "call": "DistributedOneBitAdam.step after a pinned host copy"}

    peak = measured_peaks()
    n_real = wl.n
    pack_bytes = n_real * (1 / 8 + 12 * wl_local + wl_local / 8)
    pack_ms, pack_n = prof["ob_pack_kernel"]
    pack_avg_s = pack_ms / 1e3 / max(1, pack_n)
    achieved = pack_bytes / pack_avg_s / 1e9
    per_kernel = {name: {"ms_per_step": kms / args.steps, "launches_per_step": cnt / args.steps}
                  for name, (kms, cnt) in prof.items() if cnt}
    if rank == 0:
        line = {
            "metric": METRIC, "value": wl.n / (ms_per_step / 1e3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": workload_config(wl, n_pad, f"dp{world}: split step, {wl_local} of the W={wl.W} "
                                                 "workers per GPU, "
                                                 + ("words stored and loaded by the kernels over "
                                                    "peer memory, scales over NCCL"
                                                    if D.peer_words else "per-chunk NCCL exchange"),
                                      len(grads)),
            "exchange_bytes_in_per_rank_per_step": D.exchange_bytes(),
            "roofline": {"bound": "hbm", "kernel": "ob_pack_kernel", "achieved": achieved,
                         "peak": peak["hbm_gbs"], "peak_source": peak["source"], "unit": "GB/s",
                         "frac": achieved / peak["hbm_gbs"], "traffic": None,
                         "algorithmic_bytes_per_launch": pack_bytes,
                         "avg_launch_ms": pack_avg_s * 1e3, "rank": 0},
            "kernels_rank0": per_kernel,
            "pre_path_rank0": {k: v for k, v in pre_prof.items() if v[1]},
            "cpu_baseline": None, "e2e": e2e, "gpu_launches": launches, "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    D.close()
    if world > 1:
        import torch.distributed as dist
        barrier(world)
        dist.destroy_process_group()


def run_b200(args) -> None:
    from error_compensated_bit_adam_b200.optimizer import OneBitAdam

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    multi = args.multi or ("split" if world > 1 else "single")
    if multi == "split":
        run_split(args, world, rank, dev)
        return

    wl = pick_workload(args)
    offsets, n_pad = B.ob_layout(wl.numels)
    params = WL.make_params(wl, offsets, n_pad, device=dev)
    scale = WL.grad_scale_vector(wl, offsets, n_pad, device=dev)
    opt = OneBitAdam(wl.numels, wl.W, params=params, device=dev, layerwise=args.lamb or False, **WL.HYPER)
    set_bytes = 4 * wl.W * n_pad
    free_bytes = torch.cuda.mem_get_info(dev)[0]
    n_sets = GRAD_SETS if free_bytes > GRAD_SETS * set_bytes + 2 * 4 * n_pad + (1 << 30) else 1
    grads = [torch.empty((wl.W, n_pad), dtype=torch.float32, device=dev) for _ in range(n_sets)]

    step = 0
    opt.profile(True)                          # the pre-path's kernels, by their own events
    for _ in range(wl.warmup_steps):           # full-precision Adam warmup, outside the step
        WL.fill_grads(wl, step, scale, grads[0])
        step += 1
        opt.warmup_step(grads[0])
    opt.freeze()
    pre_prof = opt.profile_read(reset=True)
    opt.profile(False)
    for gs in grads:                           # fresh draws for the timed steps
        WL.fill_grads(wl, step, scale, gs)
        step += 1
    del scale
    for k in range(args.warmup):               # untimed compressed steps
        opt.step(grads[k % n_sets])
    torch.cuda.synchronize(dev)

    stream = opt.stream

    def timed(steps: int, sample_clocks: bool):
        """K steps between CUDA events on the context's stream, barrier and
        synchronize on both sides; the slowest rank's ms per step."""
        sampler = ClockSampler()
        if sample_clocks and rank == 0:
            sampler.start()
        barrier(world)
        torch.cuda.synchronize(dev)
        sampler.mark()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for k in range(steps):
            opt.step(grads[k % n_sets])
        t1.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        clk = sampler.stop() if sample_clocks and rank == 0 else None
        return max_over_ranks(t0.elapsed_time(t1), world) / steps, clk

    # the timed region: the default call path (the step replayed as one CUDA
    # graph while the stream is not captured)
    opt.step(grads[0])                         # builds the step's graph (untimed)
    ms_per_step, clocks = timed(args.steps, True)
    # a second, profiled pass: the same steps launched kernel by kernel with
    # the library's event pairs between them, for the per-kernel times
    opt.profile(True)
    opt.profile_read(reset=True)
    direct_ms, _ = timed(args.steps, False)
    prof = opt.profile_read(reset=True)
    opt.profile(False)
    launches = sum(prof[B.ob_kernel_name(k)][1] for k in range(B.OB_K_PACK, B.OB_K_APPLY + 1))
    graph = {"ms_per_step_graph": ms_per_step, "ms_per_step_direct_launches_with_events": direct_ms,
             "note": "value is the default path (one CUDA graph per step); the per-kernel times "
                     "come from a second pass of the same steps launched one by one"}

    # roofline of the dominant kernel, from its own events over the timed region
    peak = measured_peaks()
    algo = algorithmic_bytes(wl.n, wl.W, lamb=bool(args.lamb))
    pack_ms, pack_n = prof["ob_pack_kernel"]
    pack_avg_s = pack_ms / 1e3 / max(1, pack_n)
    achieved = algo["ob_pack_kernel"] / pack_avg_s / 1e9
    step_gbs = algo["step"] / (ms_per_step / 1e3) / 1e9
    model_gbs = algo["model"] / (ms_per_step / 1e3) / 1e9
    # per kernel, per step, from the library's event pairs around each
    # launch in the profiled pass
    per_kernel = {}
    for name, (kms, cnt) in prof.items():
        if cnt:
            entry = {"ms_per_step": kms / args.steps, "launches_per_step": cnt / args.steps,
                     "share": kms / max(1e-12, sum(v[0] for v in prof.values()))}
            if name in algo:
                entry["gbs"] = algo[name] / (kms / args.steps / 1e3) / 1e9
                entry["algorithmic_bytes_per_launch"] = algo[name]
                entry["traffic"] = measured_traffic(traffic_key(name, bool(args.lamb)), wl.n, wl.W)
            per_kernel[name] = entry

    # the pre-path (full-precision Adam warmup and the freeze), timed by the
    # library's event pairs around each launch; the gradients each warmup
    # launch reads (4W bytes per parameter) are far larger than L2
    pre_path = {}
    for name in ("ob_warmup_kernel", "ob_freeze_kernel"):
        kms, cnt = pre_prof[name]
        if cnt:
            gbs = algo[name] / (kms / cnt / 1e3) / 1e9
            pre_path[name] = {"launches": cnt, "avg_launch_ms": kms / cnt, "gbs": gbs,
                              "frac_of_measured_hbm": gbs / peak["hbm_gbs"],
                              "algorithmic_bytes_per_launch": algo[name],
                              "traffic": measured_traffic(traffic_key(name, bool(args.lamb)), wl.n, wl.W)}

    # end to end: host gradients in pinned memory, copied in every step, and
    # the step's server scales read back, through ob_compressed_step_host
    e2e = ({"value": None, "unit": UNIT, "skipped": "--no-e2e"} if args.no_e2e
           else measure_e2e(opt, wl, n_pad, grads[0], args, world, dev))

    overlap = None
    if args.overlap:
        del grads
        torch.cuda.empty_cache()
        overlap = measure_overlap(wl, args, dev, world)

    split = None
    if args.split_ranks:
        opt.close()                            # release this context's device memory first
        opt.workspace = opt.params = opt._staging = None
        params = grads = None
        torch.cuda.empty_cache()
        split = measure_split_ranks(wl, args, dev)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl.W)

    if rank == 0:
        value = replica_throughput(wl.n, world, ms_per_step)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": dict(workload_config(wl, n_pad, f"replicas{world}" if world > 1 else "single GPU",
                                           n_sets),
                           optimizer=(f"1-bit LAMB (layerwise trust ratios, {args.lamb})" if args.lamb
                                      else "1-bit Adam")),
            "params_per_s_aggregate_all_workers": value * wl.W,
            "hbm_gbs_step": step_gbs,
            "hbm_frac_of_measured_peak_step": step_gbs / peak["hbm_gbs"],
            "bytes_per_param_step": algo["step"] / wl.n,
            "hbm_gbs_effective_dense_model": model_gbs,
            "hbm_frac_of_8tbs_effective_dense_model": model_gbs / NOMINAL_HBM_GBS,
            "roofline": {"bound": "hbm", "kernel": "ob_pack_kernel", "achieved": achieved,
                         "peak": peak["hbm_gbs"], "peak_source": peak["source"], "unit": "GB/s",
                         "frac": achieved / peak["hbm_gbs"],
                         "traffic": measured_traffic("ob_pack_kernel", wl.n, wl.W),
                         "algorithmic_bytes_per_launch": algo["ob_pack_kernel"],
                         "avg_launch_ms": pack_avg_s * 1e3},
            "kernels": per_kernel,
            "pre_path": pre_path,
            "graph_mode": graph,
            "overlap": overlap,
            "split_ranks": split,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    opt.close()
    if world > 1:
        import torch.distributed as dist
        barrier(world)
        dist.destroy_process_group()


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--workload", default=WL.BERT_LARGE_FLAT_W8.name)
    ap.add_argument("--n", type=int, default=0, help="flat vector of n elements instead")
    ap.add_argument("--workers", type=int, default=8, help="W for --n")
    ap.add_argument("--adam-steps", type=int, default=None, help="override warmup Adam steps")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-gradient end-to-end leg")
    ap.add_argument("--multi", choices=["split", "replicas"], default=None,
                    help="with --gpus N > 1: 'split' (default) spreads the W workers over the N "
                         "GPUs through the split step and its NCCL exchange; 'replicas' runs N "
                         "independent copies of the one-GPU step.  '--multi split' with one GPU "
                         "runs the split step's calls without an exchange")
    ap.add_argument("--peer-words", action="store_true",
                    help="with the split step on N > 1 GPUs: the kernels store and load the sign "
                         "words over peer memory (CUDA IPC) instead of NCCL moving them")
    ap.add_argument("--lamb", nargs="?", const="step", default=None, choices=["step", "frozen"],
                    help="time 1-bit LAMB (layerwise trust ratios, ob_set_layerwise) instead of 1-bit "
                         "Adam: ratios recomputed every step (step, the default) or kept at the "
                         "freeze (frozen)")
    ap.add_argument("--overlap", action="store_true",
                    help="also measure bucketed steps overlapping a synthetic backward pass")
    ap.add_argument("--split-ranks", type=int, default=0,
                    help="also run the split step as G ranks on this GPU and time each rank's share")
    ap.add_argument("--bucket-elems", type=int, default=1 << 25)
    ap.add_argument("--overlap-tokens", type=int, default=4096)
    ap.add_argument("--overlap-priority", type=int, default=0,
                    help="CUDA stream priority of the bucket streams (negative = higher)")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "b200" and not args.n:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_b200(args)


if __name__ == "__main__":
    main()
