"""The compressor entry point that allocates nothing.

Some callers cannot allocate device memory: a plugin inside a framework
whose caching allocator already holds the GPU's memory (a cudaMalloc of its
own fails there or fragments that pool), or a loop that cannot afford
cudaMalloc's implicit synchronization.  ob_onebit_compress_static serves
them: they pass only the input and the outputs, and the scratch comes from
a static device array of the library.

These tests call it through the C ABI and check it against
  * the CPU oracle's worker compressor with zero momentum and gradient and
    the error buffer set to x (then x itself is what it compresses), over
    edge sizes: empty, one element, around a sign word, around a tile, a
    ragged large vector and the largest size the scratch takes;
  * the worker stage of ob_compressed_step, the entry point that computes
    the same compression with scratch from the caller's workspace, on two
    calls in a row;
and check that a call changes neither the device's free memory nor torch's
allocator counters.  This file is collected last on purpose, so that a run
stopping at its first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from error_compensated_bit_adam_b200 import _binding as B
from error_compensated_bit_adam_b200.optimizer import OneBitAdam
import oracle

HP = dict(beta1=0.9, beta2=0.999, eps=1e-8, lr=1e-4)
SCALE_RTOL = 1e-6


def test_static_compressor_rejects_sizes_beyond_its_scratch():
    L = B.lib()
    assert L.ob_onebit_compress_static(None, B.OB_STATIC_MAX_ELEMENTS + 1, None, None,
                                       ctypes.c_void_p(256), None) == B.OB_ERR_WORKSPACE
    assert L.ob_onebit_compress_static(None, -1, None, None, ctypes.c_void_p(256),
                                       None) == B.OB_ERR_INVALID_ARG
    assert L.ob_onebit_compress_static(None, 10, None, None, ctypes.c_void_p(256),
                                       None) == B.OB_ERR_INVALID_ARG
    assert L.ob_onebit_compress_static(None, 10, None, None, None, None) == B.OB_ERR_INVALID_ARG


def sample(rng, n):
    x = rng.normal(0, 1e-3, n).astype(np.float32)
    x[rng.random(n) < 0.05] = 0.0           # sign(0) = +1
    x[rng.random(n) < 0.01] = -0.0
    return x


def compress_with_oracle(x: np.ndarray):
    """The oracle's worker stage with m = g = 0 and e_w = x: then
    x_w = fl(0 + e_w) is x (up to the sign of a zero, which the code
    ignores), so it is the compressor applied to x."""
    n = x.size
    zeros = np.zeros(n, np.float32)
    e = x.copy()
    bits, s = oracle.default().worker_compress(HP["beta1"], zeros, zeros, e)
    return bits, np.float32(s), e


def compress_with_workspace(x: np.ndarray):
    """The same compression through ob_compressed_step: one worker, m = 0,
    zero gradients and e_w = x, so the worker stage compresses x itself."""
    n = x.size
    opt = OneBitAdam([n], 1, **HP)
    g = torch.zeros((1, opt.n_padded), device="cuda")
    opt.warmup_step(g)
    opt.freeze()
    pad = np.zeros(opt.n_padded, np.float32)
    pad[:n] = x
    opt.write(B.OB_STATE_E_WORKER, 0, pad)
    opt.write(B.OB_STATE_M, 0, np.zeros(opt.n_padded, np.float32))
    opt.step(g)
    bits = opt.read(B.OB_STATE_BITS_WORKER, 0)[:(n + 31) // 32]
    scale = opt.read(B.OB_STATE_S_WORKER)[0, 0]
    err = opt.read(B.OB_STATE_E_WORKER, 0)[:n]
    opt.close()
    return bits, scale, err


class Buffers:
    """Device input and outputs of one call, the outputs filled with
    sentinels (all-ones words, NaN) so that unwritten entries show."""

    def __init__(self, x: np.ndarray):
        n = x.size
        self.n = n
        self.x = torch.from_numpy(x).cuda() if n else None
        self.bits = torch.full((max(1, (n + 31) // 32),), -1, dtype=torch.int32, device="cuda")
        self.err = torch.full((max(1, n),), float("nan"), device="cuda")
        self.scale = torch.full((1,), float("nan"), device="cuda")

    def call(self):
        B.ob_onebit_compress_static(self.x.data_ptr() if self.n else 0, self.n,
                                    self.bits.data_ptr() if self.n else 0,
                                    self.err.data_ptr() if self.n else 0,
                                    self.scale.data_ptr(), torch.cuda.current_stream().cuda_stream)

    def result(self):
        torch.cuda.synchronize()
        nw = (self.n + 31) // 32
        return (self.bits.cpu().numpy().view(np.uint32)[:nw], np.float32(self.scale.item()),
                self.err.cpu().numpy()[:self.n])


def compress_static(x: np.ndarray):
    buf = Buffers(x)
    buf.call()
    return buf.result()


def assert_same_compression(got, want, what):
    got_bits, got_s, got_e = got
    ref_bits, ref_s, ref_e = want
    assert np.array_equal(got_bits, ref_bits), f"{what}: sign words"
    assert abs(float(got_s) - float(ref_s)) <= SCALE_RTOL * float(ref_s), (what, got_s, ref_s)
    if got_s == ref_s:
        assert np.array_equal(got_e.view(np.uint32), ref_e.view(np.uint32)), f"{what}: errors"
    else:  # the scales differ in the last place: so may every error
        np.testing.assert_allclose(got_e, ref_e, rtol=0, atol=2e-6 * float(ref_s), err_msg=what)


@pytest.mark.gpu
def test_static_compressor_matches_oracle_on_edge_sizes():
    rng = np.random.default_rng(11)
    # consecutive calls, long then short and back: each reuses the scratch
    # the previous one filled
    sizes = (1, 31, 33, 4095, 4097, 1_000_003, 32, B.OB_STATIC_MAX_ELEMENTS, 4096 * 3 + 5)
    for n in sizes:
        x = sample(rng, n)
        assert_same_compression(compress_static(x), compress_with_oracle(x), f"n={n}")


@pytest.mark.gpu
def test_static_compressor_empty_input_writes_only_a_zero_scale():
    buf = Buffers(np.zeros(0, np.float32))
    buf.call()
    torch.cuda.synchronize()
    assert buf.scale.item() == 0.0
    assert buf.bits.cpu().numpy()[0] == -1          # no word written
    assert np.isnan(buf.err.cpu().numpy()[0])       # no error written


@pytest.mark.gpu
def test_static_compressor_matches_workspace_path_on_consecutive_calls():
    rng = np.random.default_rng(5)
    # two calls in a row: the second, shorter input reuses (and must not be
    # disturbed by) the scratch the first one filled
    for n in (1_000_003, 4096 * 3 + 5):
        x = sample(rng, n)
        assert_same_compression(compress_static(x), compress_with_workspace(x), f"n={n}")


@pytest.mark.gpu
def test_static_compressor_allocates_nothing():
    rng = np.random.default_rng(7)
    x = sample(rng, 1 << 22)
    buf = Buffers(x)
    buf.call()                                  # loads the library's device code here
    want = compress_with_oracle(x)
    assert_same_compression(buf.result(), want, "first call")
    buf.scale.fill_(float("nan"))
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    stats_before = (torch.cuda.memory_allocated(), torch.cuda.memory_reserved())
    buf.call()
    torch.cuda.synchronize()
    free_after = torch.cuda.mem_get_info()[0]
    stats_after = (torch.cuda.memory_allocated(), torch.cuda.memory_reserved())
    assert free_after == free_before, (free_before, free_after)
    assert stats_after == stats_before
    assert_same_compression(buf.result(), want, "second call")
