"""CPU oracle for the compression-phase step of 1-bit Adam.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference legs may import this package.  The
product package (``error_compensated_bit_adam_b200``) never imports it, and
this package never imports the product.

The arithmetic lives in ``onebit_oracle.c`` (plain single-threaded C99,
``-O2 -ffp-contract=off``); this module only builds it, loads it with
ctypes and marshals numpy arrays.  ``OracleRun`` is host-side bookkeeping
over a list of tensors: every tensor is an independent problem (per-tensor
scales, packing and server chunks), so a multi-tensor step is the
per-tensor step applied to each tensor in turn.

The same file holds the 1-bit LAMB variant (layerwise trust ratios on top
of the same compressed exchange; see the reading in onebit_oracle.c):
``lamb_warmup_step``, ``lamb_compressed_ratio``, ``lamb_apply_chunk``, and
``OracleRun(..., lamb=True)``.

Parity status: every C function is pinned by ``tests/test_oracle_pins.py``
(and the pins are shown to catch planted mistakes by
``tests/test_oracle_mutants.py``).  The LAMB functions are pinned by what
mathematics fixes (the trust ratio equals numpy's norm ratio, the step's
norm is lr * ||p||, a zero norm reduces the step to Adam's / 1-bit Adam's,
a float64 message-passing brute force); beyond that their reading of the
1-bit LAMB page, which prints no update rule, is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import List, Optional, Sequence

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "onebit_oracle.c")
LIBRARY = os.path.join(HERE, "liboracle.so")

CFLAGS = ["-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
          "-Wall", "-Wextra", "-Werror"]


def compile_source(src: str, out: str) -> str:
    """gcc a C source file into a shared object (atomic replace)."""
    tmp = out + ".tmp%d" % os.getpid()
    subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, src, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile onebit_oracle.c into liboracle.so next to it."""
    if force or not os.path.exists(LIBRARY) or os.path.getmtime(LIBRARY) < os.path.getmtime(SOURCE):
        compile_source(SOURCE, LIBRARY)
    return LIBRARY


def _f32(a: np.ndarray) -> np.ndarray:
    if a.dtype != np.float32 or not a.flags.c_contiguous:
        raise TypeError("expected a C-contiguous float32 array")
    return a


def _u32(a: np.ndarray) -> np.ndarray:
    if a.dtype != np.uint32 or not a.flags.c_contiguous:
        raise TypeError("expected a C-contiguous uint32 array")
    return a


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _ptr_array(arrays: Sequence[np.ndarray]):
    arr = (ctypes.c_void_p * max(1, len(arrays)))()
    for i, a in enumerate(arrays):
        arr[i] = a.ctypes.data
    return arr


class Oracle:
    """numpy front end of one loaded copy of the oracle library."""

    def __init__(self, path: str):
        L = ctypes.CDLL(path)
        i64, i32, f32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_void_p
        L.orc_num_words.argtypes = [i64]
        L.orc_num_words.restype = i64
        L.orc_chunk_range.argtypes = [i64, i32, i32, ctypes.POINTER(i64), ctypes.POINTER(i64)]
        L.orc_chunk_range.restype = None
        L.orc_adam_warmup_step.argtypes = [i64, i32, i32, f32, f32, f32, f32, vp, vp, vp, vp]
        L.orc_adam_warmup_step.restype = None
        L.orc_freeze.argtypes = [i64, i32, f32, f32, vp, vp]
        L.orc_freeze.restype = None
        L.orc_worker_compress.argtypes = [i64, f32, vp, vp, vp, vp, vp, ctypes.POINTER(f32)]
        L.orc_worker_compress.restype = i32
        L.orc_server_compress.argtypes = [i64, i32, vp, vp, vp, vp, vp, vp]
        L.orc_server_compress.restype = i32
        L.orc_apply.argtypes = [i64, i32, f32, vp, vp, vp, vp, vp]
        L.orc_apply.restype = None
        L.orc_server_compress_chunk.argtypes = [i64, i32, i32, vp, vp, vp, vp, ctypes.POINTER(f32),
                                                vp]
        L.orc_server_compress_chunk.restype = i32
        L.orc_apply_chunk.argtypes = [i64, i32, i32, f32, vp, f32, vp, vp, vp]
        L.orc_apply_chunk.restype = None
        L.orc_sum_squares.argtypes = [i64, vp]
        L.orc_sum_squares.restype = ctypes.c_double
        L.orc_lamb_warmup_step.argtypes = [i64, i32, i32, f32, f32, f32, f32, vp, vp, vp, vp,
                                           ctypes.POINTER(f32)]
        L.orc_lamb_warmup_step.restype = i32
        L.orc_lamb_compressed_ratio.argtypes = [i64, i32, vp, vp, vp, vp]
        L.orc_lamb_compressed_ratio.restype = f32
        L.orc_lamb_apply_chunk.argtypes = [i64, i32, i32, f32, f32, vp, f32, vp, vp, vp]
        L.orc_lamb_apply_chunk.restype = None
        self.L = L
        self.path = path

    def num_words(self, n: int) -> int:
        return int(self.L.orc_num_words(n))

    def chunk_range(self, n: int, W: int, j: int):
        b, e = ctypes.c_int64(), ctypes.c_int64()
        self.L.orc_chunk_range(n, W, j, ctypes.byref(b), ctypes.byref(e))
        return int(b.value), int(e.value)

    def adam_warmup_step(self, t: int, hp: dict, g: Sequence[np.ndarray], m: np.ndarray,
                         v: np.ndarray, p: np.ndarray) -> None:
        n = m.size
        for a in (*g, m, v, p):
            _f32(a)
            assert a.size == n
        self.L.orc_adam_warmup_step(n, len(g), t, hp["beta1"], hp["beta2"], hp["eps"], hp["lr"],
                                    _ptr_array(g), _ptr(m), _ptr(v), _ptr(p))

    def freeze(self, Tw: int, hp: dict, v: np.ndarray) -> np.ndarray:
        d = np.empty_like(_f32(v))
        self.L.orc_freeze(v.size, Tw, hp["beta2"], hp["eps"], _ptr(v), _ptr(d))
        return d

    def worker_compress(self, beta1: float, m: np.ndarray, g: np.ndarray, e: np.ndarray,
                        want_x: bool = False):
        """Returns (bits, s) or (bits, s, x); e is updated in place."""
        n = m.size
        for a in (m, g, e):
            _f32(a)
            assert a.size == n
        bits = np.zeros(self.num_words(n), np.uint32)
        x = np.empty(n, np.float32) if want_x else None
        s = ctypes.c_float()
        rc = self.L.orc_worker_compress(n, beta1, _ptr(m), _ptr(g), _ptr(e), _ptr(bits), _ptr(x),
                                        ctypes.byref(s))
        if rc != 0:
            raise MemoryError("oracle worker stage out of memory")
        return (bits, np.float32(s.value), x) if want_x else (bits, np.float32(s.value))

    def server_compress(self, bits: Sequence[np.ndarray], s, e_s: np.ndarray,
                        want_y: bool = False):
        """Returns (sbits, s_srv[W]) or (sbits, s_srv, y); e_s is updated in place."""
        n = e_s.size
        W = len(bits)
        _f32(e_s)
        for b in bits:
            _u32(b)
            assert b.size == self.num_words(n)
        s = np.ascontiguousarray(s, np.float32)
        assert s.size == W
        sbits = np.zeros(self.num_words(n), np.uint32)
        s_srv = np.zeros(W, np.float32)
        y = np.empty(n, np.float32) if want_y else None
        rc = self.L.orc_server_compress(n, W, _ptr_array(bits), _ptr(s), _ptr(e_s), _ptr(sbits),
                                        _ptr(s_srv), _ptr(y))
        if rc != 0:
            raise MemoryError("oracle server stage out of memory")
        return (sbits, s_srv, y) if want_y else (sbits, s_srv)

    def apply_update(self, lr: float, sbits: np.ndarray, s_srv, d: np.ndarray, p: np.ndarray,
                     m: np.ndarray) -> None:
        n = p.size
        for a in (d, p, m):
            _f32(a)
            assert a.size == n
        _u32(sbits)
        s_srv = np.ascontiguousarray(s_srv, np.float32)
        self.L.orc_apply(n, s_srv.size, lr, _ptr(sbits), _ptr(s_srv), _ptr(d), _ptr(p), _ptr(m))


    def server_compress_chunk(self, j: int, bits: Sequence[np.ndarray], s, e_s: np.ndarray,
                              sbits: np.ndarray) -> np.float32:
        """Server stage of chunk j only: writes chunk j's elements of e_s and
        its words of sbits; returns s'_j."""
        n = e_s.size
        s = np.ascontiguousarray(s, np.float32)
        out = ctypes.c_float()
        rc = self.L.orc_server_compress_chunk(n, len(bits), j, _ptr_array(bits), _ptr(s), _ptr(e_s),
                                              _ptr(_u32(sbits)), ctypes.byref(out), None)
        if rc != 0:
            raise MemoryError("oracle server stage out of memory")
        return np.float32(out.value)

    def apply_chunk(self, j: int, W: int, lr: float, sbits: np.ndarray, s_srv_j, d: np.ndarray,
                    p: np.ndarray, m: np.ndarray) -> None:
        self.L.orc_apply_chunk(p.size, W, j, lr, _ptr(_u32(sbits)), float(s_srv_j), _ptr(d),
                               _ptr(p), _ptr(m))


    # ----------------------------------------------------- 1-bit LAMB
    def sum_squares(self, x: np.ndarray) -> float:
        return float(self.L.orc_sum_squares(_f32(x).size, _ptr(x)))

    def lamb_warmup_step(self, t: int, hp: dict, g: Sequence[np.ndarray], m: np.ndarray,
                         v: np.ndarray, p: np.ndarray) -> np.float32:
        """One 1-bit LAMB warmup step of one tensor; returns its trust ratio."""
        n = m.size
        for a in (*g, m, v, p):
            _f32(a)
            assert a.size == n
        ratio = ctypes.c_float()
        rc = self.L.orc_lamb_warmup_step(n, len(g), t, hp["beta1"], hp["beta2"], hp["eps"],
                                         hp["lr"], _ptr_array(g), _ptr(m), _ptr(v), _ptr(p),
                                         ctypes.byref(ratio))
        if rc != 0:
            raise MemoryError("oracle LAMB warmup out of memory")
        return np.float32(ratio.value)

    def lamb_compressed_ratio(self, W: int, sbits: np.ndarray, s_srv, d: np.ndarray,
                              p: np.ndarray) -> np.float32:
        s_srv = np.ascontiguousarray(s_srv, np.float32)
        return np.float32(self.L.orc_lamb_compressed_ratio(p.size, W, _ptr(_u32(sbits)), _ptr(s_srv),
                                                           _ptr(_f32(d)), _ptr(_f32(p))))

    def lamb_apply_chunk(self, j: int, W: int, lr: float, ratio, sbits: np.ndarray, s_srv_j,
                         d: np.ndarray, p: np.ndarray, m: np.ndarray) -> None:
        self.L.orc_lamb_apply_chunk(p.size, W, j, lr, float(ratio), _ptr(_u32(sbits)),
                                    float(s_srv_j), _ptr(d), _ptr(p), _ptr(m))


_default: Optional[Oracle] = None


def default() -> Oracle:
    """The oracle built from onebit_oracle.c (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


class OracleRun:
    """The oracle's state for a list of tensors and W simulated workers.

    Per tensor t: p, m, v (then d), e_w[w], e_s; after each compressed step
    also the packed words and scales of that step.  All arrays are dense
    float32 / uint32 numpy arrays of the tensor's own length (no padding).

    threads > 1 runs independent oracle calls concurrently (ctypes releases
    the GIL): the worker stage of every (tensor, worker), the server stage
    and update of every (tensor, server chunk), and slices of the
    elementwise warmup and freeze.  Each call is still the plain single-threaded C function, so
    the results do not depend on `threads`.

    lamb=True runs 1-bit LAMB: the warmup and the update scale each
    tensor's step by its trust ratio (kept in ``ratio`` after each step);
    the warmup then runs one call per tensor, the compressed step the
    server stage of every chunk before any update.  With lamb_frozen=True
    (the other reading of the 1-bit LAMB page) the ratios are those of the
    last warmup step, kept at the freeze like the variance, and the
    compressed steps use them instead of recomputing them.
    """

    SLICE = 1 << 22  # elements per warmup/freeze call when threaded

    def __init__(self, params: Sequence[np.ndarray], W: int, hp: dict,
                 oracle: Optional[Oracle] = None, threads: int = 1, lamb: bool = False,
                 lamb_frozen: bool = False):
        if lamb_frozen and not lamb:
            raise ValueError("lamb_frozen needs lamb")
        self.lamb = bool(lamb)
        self.lamb_frozen = bool(lamb_frozen)
        self.frozen_ratio: Optional[np.ndarray] = None  # [T] the ratios kept at the freeze
        self.ratio: Optional[np.ndarray] = None  # [T] trust ratios of the last step (LAMB)
        self.threads = max(1, int(threads))
        self.o = oracle or default()
        self.W = int(W)
        self.hp = dict(hp)
        self.p = [np.array(a, np.float32, copy=True).ravel() for a in params]
        self.numel = [a.size for a in self.p]
        self.m = [np.zeros(n, np.float32) for n in self.numel]
        self.v = [np.zeros(n, np.float32) for n in self.numel]
        self.d: Optional[List[np.ndarray]] = None
        self.e_w = [[np.zeros(n, np.float32) for n in self.numel] for _ in range(self.W)]
        self.e_s = [np.zeros(n, np.float32) for n in self.numel]
        self.t_warmup = 0
        self.t_compressed = 0
        self.bits_w = None  # [w][t] words of the last step
        self.sbits = None   # [t]
        self.s_w = None     # [w, t]
        self.s_srv = None   # [t, j]

    @property
    def T(self) -> int:
        return len(self.p)

    def _run(self, jobs):
        """Run independent zero-argument callables, concurrently if threaded."""
        if self.threads == 1:
            for j in jobs:
                j()
            return
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(self.threads) as ex:
            for f in [ex.submit(j) for j in jobs]:
                f.result()

    def _slices(self, n: int):
        step = self.SLICE if self.threads > 1 else max(1, n)
        return [(a, min(n, a + step)) for a in range(0, n, step)] or [(0, 0)]

    def warmup_step(self, grads: Sequence[Sequence[np.ndarray]]) -> None:
        """grads[w][t]: worker w's gradient of tensor t."""
        assert self.d is None, "already frozen"
        self.t_warmup += 1
        t_step = self.t_warmup
        if self.lamb:  # the trust ratio needs the whole tensor: one call per tensor
            self.ratio = np.zeros(self.T, np.float32)

            def lamb_job(t):
                self.ratio[t] = self.o.lamb_warmup_step(t_step, self.hp,
                                                        [grads[w][t] for w in range(self.W)],
                                                        self.m[t], self.v[t], self.p[t])
            self._run([lambda t=t: lamb_job(t) for t in range(self.T)])
            return
        jobs = []
        for t in range(self.T):
            for a, b in self._slices(self.numel[t]):
                jobs.append(lambda t=t, a=a, b=b: self.o.adam_warmup_step(
                    t_step, self.hp, [grads[w][t][a:b] for w in range(self.W)],
                    self.m[t][a:b], self.v[t][a:b], self.p[t][a:b]))
        self._run(jobs)

    def freeze(self) -> None:
        assert self.d is None and self.t_warmup >= 1
        self.d = [np.empty_like(v) for v in self.v]

        def job(t, a, b):
            self.d[t][a:b] = self.o.freeze(self.t_warmup, self.hp, self.v[t][a:b])
        self._run([lambda t=t, a=a, b=b: job(t, a, b)
                   for t in range(self.T) for a, b in self._slices(self.numel[t])])
        if self.lamb_frozen:  # the last warmup step's trust ratios, kept
            self.frozen_ratio = np.array(self.ratio, np.float32, copy=True)
        # e_w = 0, e_s = 0 (fresh zero arrays: their pages are only touched
        # when the first compressed step writes them)
        self.e_w = [[np.zeros(n, np.float32) for n in self.numel] for _ in range(self.W)]
        self.e_s = [np.zeros(n, np.float32) for n in self.numel]

    def worker_stage(self, w: int, t: int, g: np.ndarray):
        """Worker stage of one worker on one tensor; returns (bits, s)."""
        return self.o.worker_compress(self.hp["beta1"], self.m[t], g, self.e_w[w][t])

    def compressed_step(self, grads: Sequence[Sequence[np.ndarray]]) -> None:
        """grads[w][t]: worker w's gradient of tensor t."""
        self.begin_compressed_step()
        self.worker_stages(lambda w: grads[w], range(self.W))
        self.end_compressed_step()

    # The compressed step in its phases, for callers that cannot hold every
    # worker's gradient at once: begin, then the worker stages of any
    # subsets of the workers (each worker exactly once), then the end (the
    # server stage and the update).  Same calls, same results.
    def begin_compressed_step(self) -> None:
        assert self.d is not None, "not frozen"
        T, W = self.T, self.W
        self.bits_w = [[None] * T for _ in range(W)]
        self.s_w = np.zeros((W, T), np.float32)
        self.sbits = [None] * T
        self.s_srv = np.zeros((T, W), np.float32)

    def worker_stages(self, grads_of, workers) -> None:
        """Worker stage of each worker w in `workers`, grads_of(w)[t] being
        its gradient of tensor t."""
        rows = {w: grads_of(w) for w in workers}

        def worker_job(t, w):
            b, s = self.worker_stage(w, t, rows[w][t])
            self.bits_w[w][t] = b
            self.s_w[w, t] = s

        self._run([lambda t=t, w=w: worker_job(t, w) for t in range(self.T) for w in rows])

    def end_compressed_step(self) -> None:
        T, W = self.T, self.W
        assert all(b is not None for row in self.bits_w for b in row), "a worker stage is missing"

        def server_job(t):
            sb, ss = self.o.server_compress([self.bits_w[w][t] for w in range(W)], self.s_w[:, t],
                                            self.e_s[t])
            self.sbits[t] = sb
            self.s_srv[t] = ss
            self.o.apply_update(self.hp["lr"], sb, ss, self.d[t], self.p[t], self.m[t])

        def chunk_job(t, j):  # chunks are independent: own elements, scale and words
            bits = [self.bits_w[w][t] for w in range(W)]
            self.s_srv[t, j] = self.o.server_compress_chunk(j, bits, self.s_w[:, t], self.e_s[t],
                                                            self.sbits[t])
            self.o.apply_chunk(j, W, self.hp["lr"], self.sbits[t], self.s_srv[t, j], self.d[t],
                               self.p[t], self.m[t])

        if self.lamb:  # server stage of every chunk, then each tensor's ratio, then the update
            def srv_job(t, j):
                bits = [self.bits_w[w][t] for w in range(W)]
                self.s_srv[t, j] = self.o.server_compress_chunk(j, bits, self.s_w[:, t],
                                                                self.e_s[t], self.sbits[t])

            for t in range(T):
                self.sbits[t] = np.zeros(self.o.num_words(self.numel[t]), np.uint32)
            self._run([lambda t=t, j=j: srv_job(t, j) for t in range(T) for j in range(W)])
            if self.lamb_frozen:
                self.ratio = self.frozen_ratio.copy()
            else:
                self.ratio = np.zeros(T, np.float32)

                def ratio_job(t):
                    self.ratio[t] = self.o.lamb_compressed_ratio(W, self.sbits[t], self.s_srv[t],
                                                                 self.d[t], self.p[t])
                self._run([lambda t=t: ratio_job(t) for t in range(T)])
            self._run([lambda t=t, j=j: self.o.lamb_apply_chunk(
                j, W, self.hp["lr"], self.ratio[t], self.sbits[t], self.s_srv[t, j], self.d[t],
                self.p[t], self.m[t]) for t in range(T) for j in range(W)])
            self.t_compressed += 1
            return
        if self.threads == 1:
            self._run([lambda t=t: server_job(t) for t in range(T)])
        else:
            for t in range(T):
                self.sbits[t] = np.zeros(self.o.num_words(self.numel[t]), np.uint32)
            self._run([lambda t=t, j=j: chunk_job(t, j) for t in range(T) for j in range(W)])
        self.t_compressed += 1
