"""Drives the CUDA path (through the C ABI) and the CPU oracle side by side on
the same seeded inputs.  Inputs come from error_compensated_bit_adam_b200.
workloads only; no oracle input or expected value comes from the CUDA
path, except in re-synced runs, where the state *entering* a step is copied
from the oracle INTO the GPU (never the other way)."""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch

from error_compensated_bit_adam_b200 import _binding as B
from error_compensated_bit_adam_b200 import workloads as WL
from error_compensated_bit_adam_b200.optimizer import OneBitAdam
import oracle


def to_padded(arrays, offsets, n_pad, dtype=np.float32):
    out = np.zeros(n_pad, dtype)
    for a, o in zip(arrays, offsets):
        out[o:o + a.size] = a
    return out


def words_of(flat_words: np.ndarray, offsets, numels):
    """Per-tensor word arrays out of a padded word buffer, plus a check that
    the words past each tensor's last one (its padding) are zero."""
    out = []
    for t, (o, n) in enumerate(zip(offsets, numels)):
        w0 = o // 32
        nw = (n + 31) // 32
        out.append(flat_words[w0:w0 + nw])
        pad_end = w0 + ((n + 127) // 128) * 4
        assert np.all(flat_words[w0 + nw:pad_end] == 0), f"padding words of tensor {t} not zero"
    return out


class DeviceSlices:
    """One worker's gradient of one tensor as the oracle reads it, copied
    from the device buffer that the seeded generator filled, slice by slice
    when sliced (a[a:b]) or whole (np.asarray)."""

    def __init__(self, row: torch.Tensor, offset: int, numel: int):
        self.row, self.offset, self.numel = row, offset, numel

    def __len__(self):
        return self.numel

    def __getitem__(self, sl):
        a, b, step = sl.indices(self.numel)
        assert step == 1
        return self.row[self.offset + a:self.offset + b].cpu().numpy()

    def __array__(self, dtype=None, copy=None):
        a = self[0:self.numel]
        return a if dtype is None else a.astype(dtype, copy=False)


class Pair:
    """A GPU context and an oracle run over the same workload.

    stream_workers=K keeps the host from holding every worker's gradient at
    once (for the largest workloads): the oracle's warmup reads the
    gradients slice by slice from the device buffer, and its compressed
    step runs the worker stages K workers at a time, each group's
    gradients copied to the host just before."""

    def __init__(self, wl: WL.Workload, device="cuda", threads: int = 1, hp: Optional[dict] = None,
                 lamb=False, stream_workers: Optional[int] = None):
        self.wl = wl
        self.stream = stream_workers
        self.lamb = lamb
        self.hp = dict(hp or WL.HYPER)
        self.W = wl.W
        self.numels = wl.numels
        self.offsets, self.n_pad = B.ob_layout(self.numels)
        self.dev = torch.device(device)
        params = WL.make_params(wl, self.offsets, self.n_pad, device=self.dev)
        self.scale = WL.grad_scale_vector(wl, self.offsets, self.n_pad, device=self.dev)
        # lamb: False (1-bit Adam), True or "step" (1-bit LAMB, ratios every
        # step) or "frozen" (1-bit LAMB, ratios kept at the freeze)
        self.gpu = OneBitAdam(self.numels, wl.W, params=params.clone(), layerwise=lamb, **self.hp)
        self.orc = oracle.OracleRun(WL.split(params.cpu().numpy(), self.offsets, self.numels), wl.W,
                                    self.hp, threads=threads, lamb=bool(lamb),
                                    lamb_frozen=lamb == "frozen")
        del params
        self.grads = torch.empty((wl.W, self.n_pad), dtype=torch.float32, device=self.dev)
        self.step_index = 0

    def close(self):
        self.gpu.close()

    # ------------------------------------------------------------- inputs
    def fill_grads(self):
        WL.fill_grads(self.wl, self.step_index, self.scale, self.grads)
        self.step_index += 1

    def next_grads(self):
        self.fill_grads()
        host = self.grads.cpu().numpy()
        return [WL.split(host[w], self.offsets, self.numels) for w in range(self.W)]

    def host_row(self, w: int):
        return WL.split(self.grads[w].cpu().numpy(), self.offsets, self.numels)

    # ------------------------------------------------------------- phases
    def warmup_step(self):
        if self.stream:
            self.fill_grads()
            g = [[DeviceSlices(self.grads[w], o, n) for o, n in zip(self.offsets, self.numels)]
                 for w in range(self.W)]
        else:
            g = self.next_grads()
        self.gpu.warmup_step(self.grads)
        self.orc.warmup_step(g)

    def freeze(self):
        self.gpu.freeze()
        self.orc.freeze()

    def compressed_step(self):
        if self.stream:
            self.fill_grads()
            self.gpu.step(self.grads)
            self.orc.begin_compressed_step()
            for w0 in range(0, self.W, self.stream):
                self.orc.worker_stages(self.host_row, range(w0, min(self.W, w0 + self.stream)))
            self.orc.end_compressed_step()
            return
        g = self.next_grads()
        self.gpu.step(self.grads)
        self.orc.compressed_step(g)

    def sync_into_gpu(self):
        """Copy the oracle's state into the GPU context (re-sync)."""
        o = self.orc
        pad = lambda arrs: to_padded(arrs, self.offsets, self.n_pad)
        self.gpu.write(B.OB_STATE_P, 0, pad(o.p))
        self.gpu.write(B.OB_STATE_M, 0, pad(o.m))
        self.gpu.write(B.OB_STATE_D, 0, pad(o.d))
        for w in range(self.W):
            self.gpu.write(B.OB_STATE_E_WORKER, w, pad(o.e_w[w]))
        self.gpu.write(B.OB_STATE_E_SERVER, 0, pad(o.e_s))
        if o.lamb_frozen and o.frozen_ratio is not None:   # the kept ratios are state
            self.gpu.write(B.OB_STATE_RATIO, 0, o.frozen_ratio)

    # ------------------------------------------------------------ readers
    def read_tensors(self, kind, index=0):
        return WL.split(self.gpu.read(kind, index), self.offsets, self.numels)

    # ------------------------------------------------------------ checks
    def check_warmup_exact(self):
        for kind, ref in ((B.OB_STATE_P, self.orc.p), (B.OB_STATE_M, self.orc.m),
                          (B.OB_STATE_V, self.orc.v)):
            got = self.read_tensors(kind)
            for t in range(len(ref)):
                assert np.array_equal(got[t].view(np.uint32), ref[t].view(np.uint32)), \
                    f"warmup state {kind} tensor {t} differs"

    def check_freeze_exact(self):
        got = self.read_tensors(B.OB_STATE_D)
        for t in range(len(got)):
            assert np.array_equal(got[t].view(np.uint32), self.orc.d[t].view(np.uint32)), t

    def check_compressed(self, history_exact: bool, exact_state: bool):
        """Scales to 1e-6 relative.  Worker words bit for bit when every
        earlier scale matched exactly (the words depend on the errors, which
        depend on earlier scales), server words too when this step's worker
        scales also match; otherwise at most 1e-3 of the bits may differ.
        With exact_state (re-synced run) and exact scales, the new errors,
        momentum and parameters must match bit for bit."""
        o = self.orc
        T, W = len(self.numels), self.W
        s_w = self.gpu.read(B.OB_STATE_S_WORKER)
        s_s = self.gpu.read(B.OB_STATE_S_SERVER)
        np.testing.assert_allclose(s_w, o.s_w, rtol=1e-6, atol=0)
        np.testing.assert_allclose(s_s, o.s_srv, rtol=1e-6, atol=0)
        worker_exact = np.array_equal(s_w, o.s_w)
        scales_exact = worker_exact and np.array_equal(s_s, o.s_srv)

        def compare_words(got, ref, exact, what):
            if exact:
                assert np.array_equal(got, ref), what
            else:
                diff = np.unpackbits((got ^ ref).view(np.uint8)).sum()
                assert diff <= max(1, 1e-3 * 32 * ref.size), (what, diff)

        for w in range(W):
            got = words_of(self.gpu.read(B.OB_STATE_BITS_WORKER, w), self.offsets, self.numels)
            for t in range(T):
                compare_words(got[t], o.bits_w[w][t], history_exact, f"worker {w} words, tensor {t}")
        got = words_of(self.gpu.read(B.OB_STATE_BITS_SERVER), self.offsets, self.numels)
        for t in range(T):
            compare_words(got[t], o.sbits[t], history_exact and worker_exact, f"server words, tensor {t}")
        if scales_exact and exact_state:
            for w in range(W):
                e = self.read_tensors(B.OB_STATE_E_WORKER, w)
                for t in range(T):
                    assert np.array_equal(e[t].view(np.uint32), o.e_w[w][t].view(np.uint32)), \
                        f"worker {w} error, tensor {t}"
            for kind, ref in ((B.OB_STATE_E_SERVER, o.e_s), (B.OB_STATE_M, o.m),
                              (B.OB_STATE_P, o.p)):
                got = self.read_tensors(kind)
                for t in range(T):
                    assert np.array_equal(got[t].view(np.uint32), ref[t].view(np.uint32)), \
                        f"state {kind} tensor {t}"
        return scales_exact

    def params_rel_l2(self) -> float:
        got = np.concatenate(self.read_tensors(B.OB_STATE_P)).astype(np.float64)
        ref = np.concatenate(self.orc.p).astype(np.float64)
        return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def run_schedule(wl: WL.Workload, synced: bool, warmup: Optional[int] = None,
                 compressed: Optional[int] = None, threads: int = 1, hp: Optional[dict] = None,
                 stream_workers: Optional[int] = None):
    """Warmup (checked bit for bit every step), freeze (bit for bit), then
    compressed steps: re-synced from the oracle before each step, or left to
    run free.  Returns (pair, list of per-step 'scales exact' flags)."""
    warmup = wl.warmup_steps if warmup is None else warmup
    compressed = wl.compressed_steps if compressed is None else compressed
    pr = Pair(wl, threads=threads, hp=hp, stream_workers=stream_workers)
    for _ in range(warmup):
        pr.warmup_step()
        pr.check_warmup_exact()
    pr.freeze()
    pr.check_freeze_exact()
    flags = []
    for _ in range(compressed):
        if synced:
            pr.sync_into_gpu()
        pr.compressed_step()
        history = synced or all(flags)
        flags.append(pr.check_compressed(history_exact=history, exact_state=synced))
    return pr, flags
