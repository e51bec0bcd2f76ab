"""The GPU worker stage's sign words against the definition itself (bit k
of word i is the sign of element 32i+k, 1 for x >= 0), independent of the
oracle: every sign pattern, every tail length, +-0.0 and subnormals.

The worker stage compresses x = (beta1*m + (1-beta1)*g) + e; with m and g
zero and e written as x (one worker), it compresses x itself."""
import numpy as np
import pytest
import torch

from error_compensated_bit_adam_b200 import _binding as B
from error_compensated_bit_adam_b200 import workloads as WL
from error_compensated_bit_adam_b200.optimizer import OneBitAdam

pytestmark = pytest.mark.gpu


def packbits_words(flags):
    n = flags.size
    padded = np.zeros(((n + 31) // 32) * 32, bool)
    padded[:n] = flags
    return np.packbits(padded, bitorder="little").view("<u4").astype(np.uint32)


def compress_on_gpu(values, numels, m=None, g=None):
    """One compressed step of a one-worker context whose worker stage sees
    exactly `values` (padded layout); returns (words, scales, offsets)."""
    opt = OneBitAdam(numels, 1, **WL.HYPER)
    n_pad = opt.n_padded
    zero = torch.zeros((1, n_pad), device="cuda")
    opt.warmup_step(zero)
    opt.freeze()
    opt.write(B.OB_STATE_E_WORKER, 0, values)
    opt.write(B.OB_STATE_M, 0, np.zeros(n_pad, np.float32) if m is None else m)
    grads = zero if g is None else torch.from_numpy(g.reshape(1, -1)).cuda()
    opt.step(grads)
    out = opt.read(B.OB_STATE_BITS_WORKER, 0), opt.read(B.OB_STATE_S_WORKER), opt.offsets
    opt.close()
    return out


def test_every_16_element_sign_pattern():
    pats = np.arange(1 << 16, dtype=np.uint32)
    plus = ((pats[:, None] >> np.arange(16, dtype=np.uint32)) & 1).astype(bool).ravel()
    mags = np.random.default_rng(1).uniform(0.5, 2.0, plus.size).astype(np.float32)
    x = np.where(plus, mags, -mags).astype(np.float32)
    words, _, _ = compress_on_gpu(x, [x.size])
    assert np.array_equal(words, pats[0::2] | (pats[1::2] << 16))


def test_every_tail_length_1_to_64():
    rng = np.random.default_rng(2)
    numels = list(range(1, 65)) + [127, 128, 129, 4095, 4096, 4097]
    offs, n_pad = B.ob_layout(numels)
    x = np.zeros(n_pad, np.float32)
    for o, n in zip(offs, numels):
        x[o:o + n] = rng.normal(size=n)
    words, _, _ = compress_on_gpu(x, numels)
    for o, n in zip(offs, numels):
        w0 = o // 32
        got = words[w0:w0 + ((n + 127) // 128) * 4]
        want = packbits_words(x[o:o + n] >= 0)
        assert np.array_equal(got[:want.size], want), n
        assert np.all(got[want.size:] == 0), n   # padding bits and words are 0


def test_signed_zeros_and_subnormals():
    vals = np.array([0.0, -0.0, 1e-45, -1e-45, 1e-40, -1e-40, 1.0, -1.0], np.float32)
    n = vals.size
    offs, n_pad = B.ob_layout([n])
    e = np.zeros(n_pad, np.float32)
    e[:n] = vals
    m = np.zeros(n_pad, np.float32)
    g = np.zeros(n_pad, np.float32)
    # element 1 reaches the compressor as -0.0 only if m, g and e are all -0.0
    m[1] = g[1] = e[1] = np.float32(-0.0)
    words, scales, _ = compress_on_gpu(e, [n], m=m, g=g)
    assert int(words[0]) == 0b01010111, bin(int(words[0]))
    assert scales[0, 0] > 0


def test_all_zero_and_constant_tensors():
    words, scales, offs = compress_on_gpu(np.zeros(128, np.float32), [77])
    assert scales[0, 0] == 0
    assert np.array_equal(words[:3], packbits_words(np.ones(77, bool)))
    assert words[3] == 0   # the padding word of the 128-element slot
    words, scales, offs = compress_on_gpu(np.full(1024, -0.375, np.float32), [1000])
    assert scales[0, 0] == np.float32(0.375)
    assert np.all(words[:31] == 0) and words[31] == 0
