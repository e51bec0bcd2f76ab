"""Parity at the benchmark's full sizes, in the launch configuration
bench.py times (the library chooses tiles and grids from the sizes alone).

Each workload runs at its real size with a shortened schedule.  When the
host has the RAM for the oracle's whole state, the oracle runs the same
schedule (its independent per-tensor / per-worker calls run concurrently;
where every worker's gradient would not fit on the host at once, the
oracle reads them from the device buffer a few workers, or a slice, at a
time) and every step is compared: warmup and freeze state bit for bit, packed
worker and server words bit for bit, scales within 1e-6, parameters within
1e-5 relative L2.  Otherwise (the largest sweep points on a small host) the
run is checked on sampled elements the oracle computes one by one (warmup,
freeze and the first step's worker words are elementwise) and by
properties that hold at any size (each scale is the RMS of what it
compresses; words are the signs of x = e + C(x)).
"""
import gc
import math
import os

from typing import Optional

import numpy as np
import pytest
import torch

from error_compensated_bit_adam_b200 import _binding as B
from error_compensated_bit_adam_b200 import workloads as WL
from error_compensated_bit_adam_b200.optimizer import OneBitAdam
from gpu_harness import run_schedule
import oracle

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

PARAM_TOL = 1e-5
THREADS = max(1, min(32, os.cpu_count() or 1))


def host_available() -> int:
    try:
        import psutil
        return int(psutil.virtual_memory().available)
    except Exception:
        return 0


def oracle_host_bytes(wl: WL.Workload, stream_workers: Optional[int] = None) -> int:
    # oracle: p, m, v, d, e_s + W errors; gradients of one step (W, or K
    # when streamed K workers at a time) on the host; the GPU read-backs and
    # temporaries: ~4 more vectors
    held = wl.W if stream_workers is None else min(wl.W, stream_workers)
    return 4 * wl.n * (wl.W + held + 9)


# workers whose gradients the streamed oracle holds at once
STREAM_WORKERS = 8


def shortened(wl: WL.Workload, warmup: int, compressed: int) -> WL.Workload:
    return WL.Workload(wl.name, wl.shapes, wl.W, warmup, compressed, wl.seed, wl.fan_in_scaling,
                       wl.zero_fraction)


# the headline workloads: 10 free-running compressed steps, then parameters
# within 1e-5 relative L2 (plus every step's words and scales)
FULL = {
    WL.BERT_LARGE_FLAT_W8.name: shortened(WL.BERT_LARGE_FLAT_W8, 2, 10),
    WL.ENCODER_24L_W16.name: shortened(WL.ENCODER_24L_W16, 2, 10),
    WL.RAGGED_2000_W8.name: shortened(WL.RAGGED_2000_W8, 2, 10),
}
# sweep points: one Adam step and two compressed steps each, against the
# whole oracle whenever the host has the RAM for it (test_full_size_...
# routes by oracle_host_bytes), else sampled elements and any-size
# properties
for _w in WL.sweep():
    FULL[_w.name] = shortened(_w, 1, 2)


def run_with_oracle(wl: WL.Workload, stream_workers: Optional[int] = None):
    pr, flags = run_schedule(wl, synced=False, threads=THREADS, stream_workers=stream_workers)
    try:
        rel = pr.params_rel_l2()
        assert rel <= PARAM_TOL, rel
    finally:
        pr.close()
        torch.cuda.empty_cache()


def run_sampled(wl: WL.Workload, samples: int = 1 << 16):
    """GPU run at full size, checked on sampled elements and by properties."""
    dev = torch.device("cuda")
    offs, n_pad = B.ob_layout(wl.numels)
    params = WL.make_params(wl, offs, n_pad, device=dev)
    scale = WL.grad_scale_vector(wl, offs, n_pad, device=dev)
    opt = OneBitAdam(wl.numels, wl.W, params=params, device=dev, **WL.HYPER)
    grads = torch.empty((wl.W, n_pad), dtype=torch.float32, device=dev)
    rng = np.random.default_rng(wl.seed)
    real = np.concatenate([np.arange(o, o + n) for o, n in zip(offs, wl.numels)]) \
        if wl.n_tensors > 1 else None
    pick = np.sort(rng.choice(wl.n, size=min(samples, wl.n), replace=False))
    idx = real[pick] if real is not None else pick
    idx_t = torch.from_numpy(idx).to(dev)
    o = oracle.default()
    p_s = params[idx_t].cpu().numpy().copy()
    m_s = np.zeros_like(p_s)
    v_s = np.zeros_like(p_s)
    step = 0
    for t in range(1, wl.warmup_steps + 1):
        WL.fill_grads(wl, step, scale, grads)
        step += 1
        g_s = [grads[w][idx_t].cpu().numpy().copy() for w in range(wl.W)]
        opt.warmup_step(grads)
        o.adam_warmup_step(t, WL.HYPER, g_s, m_s, v_s, p_s)
        for kind, ref in ((B.OB_STATE_P, p_s), (B.OB_STATE_M, m_s), (B.OB_STATE_V, v_s)):
            assert np.array_equal(opt.read(kind)[idx].view(np.uint32), ref.view(np.uint32)), kind
    opt.freeze()
    d_s = o.freeze(wl.warmup_steps, WL.HYPER, v_s)
    assert np.array_equal(opt.read(B.OB_STATE_D)[idx].view(np.uint32), d_s.view(np.uint32))
    assert wl.n_tensors == 1, "sampled mode is for the flat sweep vectors"
    n = wl.n
    for k in range(wl.compressed_steps):
        WL.fill_grads(wl, step, scale, grads)
        step += 1
        if k == 0:  # first step: e_w = 0, so x and its sign are elementwise
            g_s = [grads[w][idx_t].cpu().numpy().copy() for w in range(wl.W)]
        opt.step(grads)
        s_w = opt.read(B.OB_STATE_S_WORKER)[:, 0]
        for w in (0, wl.W - 1):
            words = opt.read(B.OB_STATE_BITS_WORKER, w)
            code = np.unpackbits(words.view(np.uint8), bitorder="little")[:n].astype(bool)
            e = opt.read(B.OB_STATE_E_WORKER, w)[:n].astype(np.float64)
            x = e + np.where(code, s_w[w], -s_w[w])
            rms = math.sqrt(float(np.dot(x, x)) / n)
            assert abs(rms - s_w[w]) <= 1e-6 * s_w[w], (w, rms, s_w[w])
            sure = np.abs(x) > 1e-3 * s_w[w]
            assert np.array_equal(code[sure], x[sure] >= 0)
            if k == 0:
                bits_s, _ = o.worker_compress(WL.HYPER["beta1"], m_s, g_s[w], np.zeros_like(m_s))
                want = np.unpackbits(bits_s.view(np.uint8), bitorder="little")[:idx.size]
                assert np.array_equal(code[idx], want.astype(bool)), "sampled worker signs"
        sp = opt.read(B.OB_STATE_S_SERVER)[0]
        sw = opt.read(B.OB_STATE_BITS_SERVER)
        code = np.unpackbits(sw.view(np.uint8), bitorder="little")[:n].astype(bool)
        es = opt.read(B.OB_STATE_E_SERVER)[:n].astype(np.float64)
        for j in range(wl.W):
            b, e = B.ob_chunk_range(n, wl.W, j)
            if e == b:
                assert sp[j] == 0
                continue
            y = es[b:e] + np.where(code[b:e], sp[j], -sp[j])
            rms = math.sqrt(float(np.dot(y, y)) / (e - b))
            assert abs(rms - sp[j]) <= 1e-6 * sp[j], (j, rms, sp[j])
    opt.close()
    del grads, params, scale
    torch.cuda.empty_cache()


def device_room(wl: WL.Workload):
    gc.collect()
    torch.cuda.empty_cache()
    need = B.ob_workspace_bytes(wl.numels, wl.W) + 4 * wl.n * (wl.W + 2) + (1 << 30)
    free, _ = torch.cuda.mem_get_info()
    if need > free:
        pytest.skip(f"needs {need / 1e9:.0f} GB of device memory, {free / 1e9:.0f} GB free")


@pytest.mark.parametrize("name", list(FULL))
def test_full_size_against_oracle(name):
    """The whole oracle when the host has 1.25x the RAM it needs, with the
    gradients streamed from the device a few workers at a time when they
    would not fit all at once ((2^29, 32) on a host of about 200 GB), else
    the sampled check for a flat vector."""
    wl = FULL[name]
    device_room(wl)
    avail = host_available()
    if avail >= 1.25 * oracle_host_bytes(wl):
        print(f"{name}: whole oracle, gradients of all workers on the host")
        run_with_oracle(wl)
    elif avail >= 1.25 * oracle_host_bytes(wl, STREAM_WORKERS):
        print(f"{name}: whole oracle, gradients streamed {STREAM_WORKERS} workers at a time "
              f"(host RAM {avail / 1e9:.0f} GB)")
        run_with_oracle(wl, stream_workers=STREAM_WORKERS)
    elif wl.n_tensors == 1:
        print(f"{name}: host RAM {host_available() / 1e9:.0f} GB < 1.25 x the oracle's "
              f"{oracle_host_bytes(wl) / 1e9:.0f} GB; sampled check")
        run_sampled(wl)
    else:
        pytest.skip(f"host RAM: the oracle needs ~{oracle_host_bytes(wl) / 1e9:.0f} GB")


def test_streamed_oracle_equals_whole_oracle():
    """The streamed mode (the oracle reading the gradients slice by slice in
    the warmup and a group of workers at a time in the compressed steps; 3
    workers a group, so the groups do not divide W) on a small workload:
    the same per-step checks as above, and the same oracle parameters as
    the whole mode's, bit for bit."""
    wl = WL.Workload("streamed", ((300_001,), (4_097,)), 16, 2, 3, seed=71)
    a, _ = run_schedule(wl, synced=False, threads=4, stream_workers=3)
    b, _ = run_schedule(wl, synced=False, threads=4)
    try:
        for t in range(len(wl.numels)):
            np.testing.assert_array_equal(a.orc.p[t], b.orc.p[t])
            np.testing.assert_array_equal(a.orc.sbits[t], b.orc.sbits[t])
        assert a.params_rel_l2() <= PARAM_TOL
    finally:
        a.close()
        b.close()
