"""The compressor entry point that allocates nothing.

Some callers cannot allocate device memory (a plugin inside a framework
whose caching allocator already holds the GPU's memory, or a loop that
cannot afford cudaMalloc's implicit synchronization).
ob_onebit_compress_static serves them: they pass only the input and the
outputs, and the scratch comes from a static device array of the library.
These tests check it through the C ABI against the worker stage of
ob_compressed_step, which computes the same compression with scratch from
the caller's workspace.  This file is collected last on purpose, so that a
run stopping at its first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from error_compensated_bit_adam_b200 import _binding as B
from error_compensated_bit_adam_b200.optimizer import OneBitAdam

HP = dict(beta1=0.9, beta2=0.999, eps=1e-8, lr=1e-4)


def test_static_compressor_rejects_sizes_beyond_its_scratch():
    L = B.lib()
    assert L.ob_onebit_compress_static(None, B.OB_STATIC_MAX_ELEMENTS + 1, None, None,
                                       ctypes.c_void_p(256), None) == B.OB_ERR_WORKSPACE
    assert L.ob_onebit_compress_static(None, -1, None, None, ctypes.c_void_p(256),
                                       None) == B.OB_ERR_INVALID_ARG
    assert L.ob_onebit_compress_static(None, 10, None, None, ctypes.c_void_p(256),
                                       None) == B.OB_ERR_INVALID_ARG
    assert L.ob_onebit_compress_static(None, 10, None, None, None, None) == B.OB_ERR_INVALID_ARG


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


def compress_static(x: np.ndarray):
    n = x.size
    dx = torch.from_numpy(x).cuda()
    bits = torch.full(((n + 31) // 32,), -1, dtype=torch.int32, device="cuda")
    err = torch.full((n,), float("nan"), device="cuda")
    scale = torch.full((1,), float("nan"), device="cuda")
    stream = torch.cuda.current_stream()
    B.ob_onebit_compress_static(dx.data_ptr(), n, bits.data_ptr(), err.data_ptr(),
                                scale.data_ptr(), stream.cuda_stream)
    torch.cuda.synchronize()
    return (bits.cpu().numpy().view(np.uint32), np.float32(scale.item()), err.cpu().numpy())


@pytest.mark.gpu
def test_static_compressor_matches_workspace_path_on_consecutive_calls():
    rng = np.random.default_rng(5)
    # two calls in a row: the second, shorter input reuses (and must not be
    # disturbed by) the scratch the first one filled
    for n in (1_000_003, 4096 * 3 + 5):
        x = rng.normal(0, 1e-3, n).astype(np.float32)
        x[rng.random(n) < 0.05] = 0.0
        got_bits, got_s, got_e = compress_static(x)
        ref_bits, ref_s, ref_e = compress_with_workspace(x)
        assert np.array_equal(got_bits, ref_bits)
        assert abs(float(got_s) - float(ref_s)) <= 1e-6 * float(ref_s)
        if got_s == ref_s:
            assert np.array_equal(got_e.view(np.uint32), ref_e.view(np.uint32))
        else:
            np.testing.assert_allclose(got_e, ref_e, rtol=0, atol=2e-6 * float(ref_s))
