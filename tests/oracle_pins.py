"""Pins of the CPU oracle: each check compares the oracle against something
other than itself.

* torch.optim.Adam / torch.optim.SGD (library routines) for the warmup, the
  freeze and the W=1 lossless case;
* numpy's bit packing and norms for the 1-bit code;
* exhaustive sign patterns, special values (+-0, subnormals, constants);
* invariants: the error feedback telescopes, W=1 server is the identity,
  identical workers give W-independent results;
* a message-passing brute force in float64 for tiny tensors;
* closed forms for the server chunks and the communication volume.

Every function takes an ``oracle.Oracle`` so tests/test_oracle_mutants.py
can run the same pins against copies of the oracle with planted mistakes.
A pin raises AssertionError on failure.

Cited passages are on the review page "1-bit Adam: Communication Efficient
Large-Scale Training with Adam's Convergence Speed" ([1BA]).
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch

HP = dict(beta1=0.9, beta2=0.999, eps=1e-8, lr=1e-4)
F32 = np.float32
F64 = np.float64
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def hp32(key: str) -> float:
    """The float32 value of a hyperparameter, as a Python float."""
    return float(F32(HP[key]))


def packbits_words(flags: np.ndarray) -> np.ndarray:
    """numpy's little-endian packing: bit k of word i is flags[32 i + k]."""
    n = flags.size
    nw = (n + 31) // 32
    padded = np.zeros(nw * 32, bool)
    padded[:n] = flags
    return np.packbits(padded, bitorder="little").view("<u4").astype(np.uint32)


def unpack_words(words: np.ndarray, n: int) -> np.ndarray:
    return np.unpackbits(np.ascontiguousarray(words, "<u4").view(np.uint8),
                         bitorder="little")[:n].astype(bool)


def ulp(x) -> np.ndarray:
    return np.spacing(np.abs(np.asarray(x, F32))).astype(F64)


# ---------------------------------------------------------------------------
# warmup and freeze against torch.optim.Adam       [1BA, Proposed method, 1]
# ---------------------------------------------------------------------------

def pin_warmup_matches_torch_adam(o, W=3, steps=6, n=1001, seed=1):
    rng = np.random.default_rng(seed)
    p = rng.normal(0, 0.02, n).astype(F32)
    tp = torch.nn.Parameter(torch.from_numpy(p.copy()))
    opt = torch.optim.Adam([tp], lr=hp32("lr"), betas=(hp32("beta1"), hp32("beta2")),
                           eps=hp32("eps"), foreach=False)
    m = np.zeros(n, F32)
    v = np.zeros(n, F32)
    zero = rng.random(n) < 0.1
    for t in range(1, steps + 1):
        g = [np.where(zero, 0.0, rng.normal(0, 1e-3, n)).astype(F32) for _ in range(W)]
        o.adam_warmup_step(t, HP, g, m, v, p)
        tp.grad = torch.from_numpy((np.sum(np.stack(g).astype(F64), 0) / W).astype(F32))
        opt.step()
    st = opt.state[tp]
    np.testing.assert_allclose(m, st["exp_avg"].numpy(), rtol=3e-6, atol=1e-11)
    np.testing.assert_allclose(v, st["exp_avg_sq"].numpy(), rtol=3e-6, atol=1e-17)
    np.testing.assert_allclose(p, tp.detach().numpy(), rtol=3e-6, atol=2e-9)
    assert np.all(m[zero] == 0) and np.all(v[zero] == 0)


def pin_freeze_is_last_adam_denominator(o, steps=5, n=513, seed=2):
    """[1BA, Abstract; Proposed method, 2]: the frozen preconditioner is the
    denominator Adam used at its last warmup step."""
    rng = np.random.default_rng(seed)
    tp = torch.nn.Parameter(torch.from_numpy(rng.normal(0, 0.02, n).astype(F32)))
    opt = torch.optim.Adam([tp], lr=hp32("lr"), betas=(hp32("beta1"), hp32("beta2")),
                           eps=hp32("eps"), foreach=False)
    for _ in range(steps):
        tp.grad = torch.from_numpy(rng.normal(0, 1e-3, n).astype(F32))
        opt.step()
    v = opt.state[tp]["exp_avg_sq"]
    bc2 = 1.0 - hp32("beta2") ** steps
    denom = (v.sqrt() / math.sqrt(bc2)).add_(hp32("eps")).numpy()
    d = o.freeze(steps, HP, np.ascontiguousarray(v.numpy()))
    np.testing.assert_allclose(d, denom, rtol=2e-6, atol=0)


# ---------------------------------------------------------------------------
# the 1-bit code                                     [1BA, Abstract]
# ---------------------------------------------------------------------------

def _compress_values(o, x: np.ndarray, want_x=False):
    """Worker stage with m = g = 0 and e = x, so the stage compresses x
    itself (x = (0 + 0) + e is exact; -0.0 becomes +0.0)."""
    z = np.zeros(x.size, F32)
    e = np.ascontiguousarray(x, F32).copy()
    out = o.worker_compress(HP["beta1"], z, z.copy(), e, want_x=want_x)
    return (*out, e)


def pin_packing_matches_numpy(o, seed=3):
    rng = np.random.default_rng(seed)
    for n in list(range(1, 65)) + [100, 127, 128, 129, 1000, 4097]:
        x = rng.normal(0, 1, n).astype(F32)
        bits, s, _ = _compress_values(o, x)
        assert bits.size == (n + 31) // 32
        assert np.array_equal(bits, packbits_words(x >= 0)), n


def pin_exhaustive_sign_patterns(o, seed=4):
    """Every sign pattern of k <= 12 elements: the single packed word equals
    the pattern read as a binary number (element j <-> bit j)."""
    rng = np.random.default_rng(seed)
    for k in range(1, 13):
        mags = rng.uniform(0.5, 2.0, k).astype(F32)
        for pat in range(1 << k):
            plus = ((pat >> np.arange(k)) & 1).astype(bool)
            bits, _, _ = _compress_values(o, np.where(plus, mags, -mags).astype(F32))
            assert bits.size == 1 and int(bits[0]) == pat, (k, pat)
    # all 2^16 patterns of 16 elements back to back: word i = pattern 2i | pattern 2i+1 << 16
    pats = np.arange(1 << 16, dtype=np.uint32)
    plus = ((pats[:, None] >> np.arange(16, dtype=np.uint32)) & 1).astype(bool).ravel()
    mags = rng.uniform(0.5, 2.0, plus.size).astype(F32)
    bits, _, _ = _compress_values(o, np.where(plus, mags, -mags).astype(F32))
    assert np.array_equal(bits, pats[0::2] | (pats[1::2] << 16))


def pin_sign_rule_and_special_values(o):
    """sign(0) = +1 for +0.0 and -0.0; subnormals keep their sign; an
    all-zero tensor has scale 0 and all codes +1; a constant tensor c has
    scale |c| and zero error."""
    vals = np.array([0.0, -0.0, 1e-45, -1e-45, 1e-40, -1e-40, 1.0, -1.0], F32)
    n = vals.size
    # element 1 must reach the compressor as -0.0: m = g = e = -0.0 there
    m = np.zeros(n, F32)
    g = np.zeros(n, F32)
    e = vals.copy()
    m[1] = g[1] = e[1] = F32(-0.0)
    bits, s, x = o.worker_compress(HP["beta1"], m, g, e, want_x=True)
    assert np.signbit(x[1]) and x[1] == 0, "the -0.0 case did not reach the compressor"
    assert int(bits[0]) == 0b01010111, bin(int(bits[0]))
    for n in (1, 31, 77):
        bits, s, e = _compress_values(o, np.zeros(n, F32))
        assert s == 0 and np.all(e == 0)
        assert np.array_equal(bits, packbits_words(np.ones(n, bool)))
    for c in (0.375, -0.375, 3.0):
        bits, s, e = _compress_values(o, np.full(1000, c, F32))
        assert s == F32(abs(c)) and np.all(e == 0)
        assert np.array_equal(bits, packbits_words(np.full(1000, c >= 0)))


def pin_compressor_is_scale_times_sign(o, n=5000, seed=5):
    """C(x) = s * sign(x) with s = ||x||_2 / sqrt(n): decoding the words
    gives exactly +-s, e is x - C(x) correctly rounded, ||C(x)|| = ||x||, and
    x is the momentum plus the old error."""
    rng = np.random.default_rng(seed)
    m = rng.normal(0, 1e-3, n).astype(F32)
    g = rng.normal(0, 1e-3, n).astype(F32)
    e0 = rng.normal(0, 3e-4, n).astype(F32)
    e = e0.copy()
    bits, s, x = o.worker_compress(HP["beta1"], m, g, e, want_x=True)
    b1 = F64(F32(HP["beta1"]))
    x64 = b1 * m.astype(F64) + (1 - b1) * g.astype(F64) + e0.astype(F64)
    assert np.all(np.abs(x.astype(F64) - x64) <= 3 * ulp(x) + 2 * ulp(e0)), "x != beta1 m + c1 g + e"
    code = unpack_words(bits, n)
    assert np.array_equal(code, x >= 0)
    dec = np.where(code, s, -s).astype(F32)
    assert np.all(np.abs(dec) == s)
    assert np.array_equal(e, (x.astype(F64) - dec.astype(F64)).astype(F32)), "e != fl(x - C(x))"
    norm_x = np.linalg.norm(x.astype(F64))
    assert abs(F64(s) * math.sqrt(n) - norm_x) <= 2e-7 * norm_x, "scale does not keep the norm"
    assert abs(F64(s) - norm_x / math.sqrt(n)) <= 1.0 * ulp(s), "scale is not the rounded RMS"


# ---------------------------------------------------------------------------
# error feedback                                   [1BA, Proposed method, 3]
# ---------------------------------------------------------------------------

def pin_error_feedback_telescopes(o, n=3000, W=4, steps=10, seed=6):
    """Over K steps, sum_k C(x_k) + e_K = sum_k m_w,k + e_0 for each worker,
    and sum_k C_s(y_k) + e_s,K = sum_k avg_k + e_s,0 for the server, up to the
    roundings of the steps (bounded elementwise)."""
    rng = np.random.default_rng(seed)
    b1 = F64(F32(HP["beta1"]))
    e_w = [rng.normal(0, 1e-4, n).astype(F32) for _ in range(W)]
    e0_w = [e.astype(F64) for e in e_w]
    e_s = rng.normal(0, 1e-4, n).astype(F32)
    e0_s = e_s.astype(F64)
    lhs_w = [np.zeros(n) for _ in range(W)]
    rhs_w = [e.copy() for e in e0_w]
    bound_w = [np.zeros(n) for _ in range(W)]
    lhs_s, rhs_s, bound_s = np.zeros(n), e0_s.copy(), np.zeros(n)
    for _ in range(steps):
        m = rng.normal(0, 1e-3, n).astype(F32)
        bits, scales = [], []
        for w in range(W):
            g = rng.normal(0, 1e-3, n).astype(F32)
            e_prev = e_w[w].copy()
            b, s, x = o.worker_compress(HP["beta1"], m, g, e_w[w], want_x=True)
            dec = np.where(unpack_words(b, n), s, -s).astype(F64)
            mw = b1 * m.astype(F64) + (1 - b1) * g.astype(F64)
            lhs_w[w] += dec
            rhs_w[w] += mw
            bound_w[w] += 2 * ulp(mw) + ulp(x) + ulp(e_w[w]) + ulp(e_prev)
            bits.append(b)
            scales.append(s)
        e_prev_s = e_s.copy()
        sb, ss, y = o.server_compress(bits, np.array(scales, F32), e_s, want_y=True)
        avg = sum(np.where(unpack_words(bits[w], n), F64(scales[w]), -F64(scales[w]))
                  for w in range(W)) / W
        srv_scale = np.zeros(n)
        for j in range(W):
            b_, e_ = o.chunk_range(n, W, j)
            srv_scale[b_:e_] = ss[j]
        lhs_s += np.where(unpack_words(sb, n), srv_scale, -srv_scale)
        rhs_s += avg
        bound_s += W * ulp(avg) + ulp(y) + ulp(e_s) + ulp(e_prev_s)
    for w in range(W):
        resid = lhs_w[w] + e_w[w].astype(F64) - rhs_w[w]
        assert np.all(np.abs(resid) <= bound_w[w]), "worker error feedback does not telescope"
    resid = lhs_s + e_s.astype(F64) - rhs_s
    assert np.all(np.abs(resid) <= bound_s), "server error feedback does not telescope"


# ---------------------------------------------------------------------------
# W = 1 special cases                         [1BA, Proposed method, 1-2]
# ---------------------------------------------------------------------------

def pin_w1_lossless_is_preconditioned_momentum_sgd(o, steps=8, seed=7):
    """With one worker and inputs whose magnitude is constant (n = 32, so the
    double sum of squares is exact), 1-bit compression loses nothing: both
    errors stay exactly 0 and the compressed phase is momentum SGD
    preconditioned by the frozen d, as torch.optim.SGD computes it
    (momentum = dampening = beta1, gradient g/d)."""
    n = 32
    rng = np.random.default_rng(seed)
    sig = np.where(rng.random(n) < 0.5, 1.0, -1.0)
    m = (sig * 1e-3).astype(F32)
    d = (np.sqrt(rng.uniform(1e-7, 1e-5, n)) + 1e-8).astype(F32)
    p = rng.normal(0, 0.02, n).astype(F32)
    tp = torch.nn.Parameter(torch.from_numpy(p.copy()))
    b1 = hp32("beta1")
    opt = torch.optim.SGD([tp], lr=hp32("lr"), momentum=b1, dampening=b1)
    opt.state[tp]["momentum_buffer"] = torch.from_numpy(m / d)
    e_w = np.zeros(n, F32)
    e_s = np.zeros(n, F32)
    for k in range(steps):
        mag = F32(abs(m[0]))
        if k % 3 == 1:   # flip every sign: (1 - beta1) * A > beta1 * |m|
            g = (-np.sign(m) * mag * 20).astype(F32)
        else:
            g = (np.sign(m) * mag * F32(rng.uniform(0.1, 3.0))).astype(F32)
        bits, s = o.worker_compress(HP["beta1"], m, g, e_w)
        sb, ss = o.server_compress([bits], np.array([s], F32), e_s)
        o.apply_update(HP["lr"], sb, ss, d, p, m)
        assert np.all(e_w == 0) and np.all(e_s == 0), "compression of a constant-magnitude x lost data"
        tp.grad = torch.from_numpy(g / d)
        opt.step()
    np.testing.assert_allclose(p, tp.detach().numpy(), rtol=3e-6, atol=2e-9)
    np.testing.assert_allclose(m / d, opt.state[tp]["momentum_buffer"].numpy(), rtol=1e-5)


def pin_w1_server_is_identity(o, n=5000, seed=8):
    """One worker, fresh server error: the server re-compresses +-s, so
    s' = s exactly, the server code equals the worker code, and e_s = 0."""
    rng = np.random.default_rng(seed)
    m = rng.normal(0, 1e-3, n).astype(F32)
    g = rng.normal(0, 1e-3, n).astype(F32)
    e = rng.normal(0, 1e-4, n).astype(F32)
    bits, s = o.worker_compress(HP["beta1"], m, g, e)
    e_s = np.zeros(n, F32)
    sb, ss = o.server_compress([bits], np.array([s], F32), e_s)
    assert ss.size == 1 and ss[0] == s
    assert np.array_equal(sb, bits)
    assert np.all(e_s == 0)


def pin_identical_workers(o, n=100, steps=3, seed=9):
    """All workers send the same gradient.  For n <= 128 the whole tensor is
    server 0's chunk for any W, so W = 1 and W = 2 agree bit for bit (the
    sum of two equal terms and the halving are exact) and W = 4, 8 agree to
    rounding."""
    rng = np.random.default_rng(seed)
    p0 = rng.normal(0, 0.02, n).astype(F32)
    m0 = rng.normal(0, 1e-3, n).astype(F32)
    d = (np.sqrt(rng.uniform(1e-7, 1e-5, n)) + 1e-8).astype(F32)
    grads = [rng.normal(0, 1e-3, n).astype(F32) for _ in range(steps)]
    out = {}
    for W in (1, 2, 4, 8):
        p, m = p0.copy(), m0.copy()
        e_w = [np.zeros(n, F32) for _ in range(W)]
        e_s = np.zeros(n, F32)
        for k in range(steps):
            bs, ss = [], []
            for w in range(W):
                b, s = o.worker_compress(HP["beta1"], m, grads[k], e_w[w])
                bs.append(b)
                ss.append(s)
            sb, srv = o.server_compress(bs, np.array(ss, F32), e_s)
            o.apply_update(HP["lr"], sb, srv, d, p, m)
        out[W] = (p, m, e_s)
    for a, b in zip(out[1], out[2]):
        assert np.array_equal(a, b), "W=2 with identical workers differs from W=1"
    for W in (4, 8):
        np.testing.assert_allclose(out[W][0], out[1][0], rtol=1e-6, atol=1e-10)
        np.testing.assert_allclose(out[W][1], out[1][1], rtol=1e-5, atol=1e-12)


# ---------------------------------------------------------------------------
# server chunks                                    [1BA, Proposed method, 4]
# ---------------------------------------------------------------------------

def pin_chunk_layout(o):
    """Chunks tile [0, n) in order; each starts on a 128-element boundary (no
    sign word or 16-byte word group straddles two servers); every chunk but
    the trailing ones has L = roundup(ceil(n/W), 128) elements."""
    for W in (1, 2, 3, 4, 5, 7, 8, 16, 31, 32, 64):
        for n in (0, 1, 31, 32, 33, 127, 128, 129, 1000, 4095, 4096, 4097, 100_003, 1 << 20,
                  335_544_320):
            L = -(-(-(-n // W)) // 128) * 128 if n else 0
            pos = 0
            for j in range(W):
                b, e = o.chunk_range(n, W, j)
                assert b == pos and e >= b, (n, W, j)
                assert b % 128 == 0 or b == n, (n, W, j)
                assert e - b == min(L, max(0, n - j * L)), (n, W, j, e - b, L)
                pos = e
            assert pos == n


# ---------------------------------------------------------------------------
# message-passing brute force (float64)        [1BA, Proposed method, 3-4]
# ---------------------------------------------------------------------------

def _pack_bytes(codes: np.ndarray) -> bytes:
    """Pack +1/-1 codes as bits with plain integer arithmetic."""
    out = bytearray()
    for k in range(0, codes.size, 32):
        word = 0
        for i, c in enumerate(codes[k:k + 32]):
            if c > 0:
                word |= 1 << i
        out += word.to_bytes(4, "little")
    return bytes(out)


def _unpack_bytes(buf: bytes, count: int) -> np.ndarray:
    codes = []
    for i in range(count):
        word = int.from_bytes(buf[4 * (i // 32):4 * (i // 32) + 4], "little")
        codes.append(1.0 if (word >> (i % 32)) & 1 else -1.0)
    return np.array(codes, F64)


def brute_force_step(W, m, d, p, grads, e_w, e_s, lamb=False, lr=None, ratio=None):
    """One compressed step as W workers and W servers exchanging byte
    messages, in float64.  Returns a dict of results and the bytes sent.
    lamb: the update is 1-bit LAMB's, scaled by the trust ratio
    ||p|| / ||m_hat / d|| (1 when a norm is 0), or by `ratio` when given
    (the ratio kept at the freeze)."""
    n = m.size
    b1 = F64(F32(HP["beta1"]))
    lr = F64(F32(HP["lr"] if lr is None else lr))
    # chunk plan: roundup(ceil(n/W), 128) elements per server, in order
    L = -(-(-(-n // W)) // 128) * 128 if n else 0
    chunks = [(min(n, j * L), min(n, (j + 1) * L)) for j in range(W)]
    wire = 0
    outbox = {}
    res = dict(codes=[], scales=[], e_w=[])
    for w in range(W):
        x = b1 * m + (1 - b1) * grads[w] + e_w[w]
        s = math.sqrt(np.mean(x * x)) if n else 0.0
        code = np.where(x >= 0, 1.0, -1.0)
        res["codes"].append(code)
        res["scales"].append(s)
        res["e_w"].append(x - s * code)
        for j, (b, e) in enumerate(chunks):
            outbox[(w, j)] = (_pack_bytes(code[b:e]), s)
            if j != w:
                wire += len(outbox[(w, j)][0]) + 4
    bcast = {}
    res["srv_scales"], res["srv_codes"], res["e_s"] = [], np.zeros(n), np.zeros(n)
    for j, (b, e) in enumerate(chunks):
        inbox = [outbox[(w, j)] for w in range(W)]
        avg = sum(s * _unpack_bytes(buf, e - b) for buf, s in inbox) / W
        y = avg + e_s[b:e]
        s2 = math.sqrt(np.mean(y * y)) if e > b else 0.0
        code = np.where(y >= 0, 1.0, -1.0)
        res["srv_scales"].append(s2)
        res["srv_codes"][b:e] = code
        res["e_s"][b:e] = y - s2 * code
        bcast[j] = (_pack_bytes(code), s2)
        wire += (W - 1) * (len(bcast[j][0]) + 4)
    m_hat = np.zeros(n)
    for j, (b, e) in enumerate(chunks):
        buf, s2 = bcast[j]
        m_hat[b:e] = s2 * _unpack_bytes(buf, e - b)
    u = m_hat / d
    given, ratio = ratio, 1.0
    if lamb and given is not None:
        ratio = F64(given)
    elif lamb and np.linalg.norm(p) > 0 and np.linalg.norm(u) > 0:
        ratio = np.linalg.norm(p) / np.linalg.norm(u)
    res["ratio"] = ratio
    res["p"] = p - lr * ratio * u
    res["m"] = m_hat
    res["wire_bytes"] = wire
    return res


def pin_brute_force_message_passing(o, seed=10):
    rng = np.random.default_rng(seed)
    for W in (1, 2, 3, 5, 8):
        for n in (1, 5, 31, 32, 33, 64, 200, 300):
            p = rng.normal(0, 0.02, n).astype(F32)
            m = rng.normal(0, 1e-3, n).astype(F32)
            d = (np.sqrt(rng.uniform(1e-7, 1e-5, n)) + 1e-8).astype(F32)
            e_w = [rng.normal(0, 2e-4, n).astype(F32) for _ in range(W)]
            e_s = rng.normal(0, 2e-4, n).astype(F32)
            for _ in range(3):
                grads = [rng.normal(0, 1e-3, n).astype(F32) for _ in range(W)]
                ref = brute_force_step(W, m.astype(F64), d.astype(F64), p.astype(F64),
                                       [g.astype(F64) for g in grads],
                                       [e.astype(F64) for e in e_w], e_s.astype(F64))
                bits, scales, xs = [], [], []
                for w in range(W):
                    b, s, x = o.worker_compress(HP["beta1"], m, grads[w], e_w[w], want_x=True)
                    bits.append(b)
                    scales.append(s)
                    xs.append(x)
                sb, ss, y = o.server_compress(bits, np.array(scales, F32), e_s, want_y=True)
                o.apply_update(HP["lr"], sb, ss, d, p, m)
                for w in range(W):
                    sure = np.abs(xs[w]) > 1e-4 * max(scales[w], 1e-30)
                    assert np.array_equal(unpack_words(bits[w], n)[sure], ref["codes"][w][sure] > 0)
                    assert abs(scales[w] - ref["scales"][w]) <= 1e-6 * ref["scales"][w]
                    np.testing.assert_allclose(e_w[w], ref["e_w"][w], rtol=1e-4, atol=1e-9)
                np.testing.assert_allclose(ss, ref["srv_scales"], rtol=1e-5, atol=1e-12)
                sure = np.abs(y) > 1e-4 * max(float(np.max(ss)), 1e-30)
                assert np.array_equal(unpack_words(sb, n)[sure], ref["srv_codes"][sure] > 0)
                np.testing.assert_allclose(m, ref["m"], rtol=1e-5, atol=1e-12)
                np.testing.assert_allclose(p, ref["p"], rtol=1e-6, atol=1e-9)
                np.testing.assert_allclose(e_s, ref["e_s"], rtol=1e-4, atol=1e-9)


# ---------------------------------------------------------------------------
# 1-bit LAMB: layerwise trust ratios  (the 1-bit LAMB review page, Abstract)
# ---------------------------------------------------------------------------

LAMB_LR = 0.05  # large enough that p_new - p_old is far above p's rounding


def pin_lamb_warmup_from_zero_params_is_adam(o, W=3, n=777, seed=21):
    """With p = 0 the trust ratio is 1 by LAMB's convention, so the first
    LAMB warmup step is textbook Adam's first step (torch.optim.Adam)."""
    rng = np.random.default_rng(seed)
    p = np.zeros(n, F32)
    tp = torch.nn.Parameter(torch.zeros(n))
    opt = torch.optim.Adam([tp], lr=hp32("lr"), betas=(hp32("beta1"), hp32("beta2")),
                           eps=hp32("eps"), foreach=False)
    g = [rng.normal(0, 1e-3, n).astype(F32) for _ in range(W)]
    m = np.zeros(n, F32)
    v = np.zeros(n, F32)
    ratio = o.lamb_warmup_step(1, HP, g, m, v, p)
    assert ratio == 1.0, ratio
    tp.grad = torch.from_numpy((np.sum(np.stack(g).astype(F64), 0) / W).astype(F32))
    opt.step()
    np.testing.assert_allclose(m, opt.state[tp]["exp_avg"].numpy(), rtol=3e-6, atol=1e-11)
    np.testing.assert_allclose(v, opt.state[tp]["exp_avg_sq"].numpy(), rtol=3e-6, atol=1e-17)
    np.testing.assert_allclose(p, tp.detach().numpy(), rtol=3e-6, atol=2e-9)


def _adam_direction(m, v, t):
    """Adam's update direction from its moments, in float64."""
    b1, b2, eps = F64(F32(HP["beta1"])), F64(F32(HP["beta2"])), F64(F32(HP["eps"]))
    mh = m.astype(F64) / (1 - b1 ** t)
    vh = v.astype(F64) / (1 - b2 ** t)
    return mh / (np.sqrt(vh) + eps)


def pin_lamb_warmup_layerwise_step(o, W=2, n=3000, steps=4, seed=22):
    """LAMB's layerwise step, from its definition: the trust ratio equals
    numpy's ||p|| / ||r|| with r Adam's direction, the step is -lr ratio r,
    so its norm is lr ||p|| whatever the gradients; two tensors that differ
    only by a factor 10 in p take steps that differ by the same factor."""
    rng = np.random.default_rng(seed)
    hp = dict(HP, lr=LAMB_LR)
    lr = F64(F32(LAMB_LR))
    base = rng.normal(0, 0.02, n).astype(F32)
    ps = [base.copy(), (base * F32(10)).astype(F32)]
    ms = [np.zeros(n, F32) for _ in ps]
    vs = [np.zeros(n, F32) for _ in ps]
    for t in range(1, steps + 1):
        g = [rng.normal(0, 1e-3, n).astype(F32) for _ in range(W)]
        steps_norm = []
        for k in range(2):
            before = ps[k].astype(F64)
            ratio = o.lamb_warmup_step(t, hp, g, ms[k], vs[k], ps[k])
            r = _adam_direction(ms[k], vs[k], t)
            want = np.linalg.norm(before) / np.linalg.norm(r)
            assert abs(F64(ratio) - want) <= 1e-6 * want, (t, k, ratio, want)
            delta = ps[k].astype(F64) - before
            np.testing.assert_allclose(delta, -lr * F64(ratio) * r, rtol=1e-4,
                                       atol=4 * float(np.max(ulp(ps[k]))))
            norm = np.linalg.norm(delta)
            assert abs(norm - lr * np.linalg.norm(before)) <= 1e-5 * lr * np.linalg.norm(before)
            steps_norm.append(norm)
        assert abs(steps_norm[1] / steps_norm[0] - 10.0) <= 1e-4


def _server_inputs(rng, n, W):
    o_bits = rng.integers(0, 2 ** 32, (n + 31) // 32, dtype=np.uint64).astype(np.uint32)
    if n % 32:
        o_bits[-1] &= np.uint32((1 << (n % 32)) - 1)
    s_srv = rng.uniform(1e-4, 1e-3, W).astype(F32)
    d = (np.sqrt(rng.uniform(1e-7, 1e-5, n)) + 1e-8).astype(F32)
    return o_bits, s_srv, d


def pin_lamb_compressed_update(o, seed=23):
    """The compression phase's LAMB update of one tensor from given server
    words and chunk scales: m_hat decoded independently (numpy bits), the
    ratio equal to numpy's ||p|| / ||m_hat / d||, the step -lr ratio
    m_hat/d with norm lr ||p||, m = m_hat exactly; with p = 0 the ratio is
    1 and the update is 1-bit Adam's bit for bit."""
    rng = np.random.default_rng(seed)
    lr = F64(F32(LAMB_LR))
    for W, n in ((1, 100), (3, 1000), (8, 5000), (16, 130)):
        sbits, s_srv, d = _server_inputs(rng, n, W)
        code = np.where(unpack_words(sbits, n), 1.0, -1.0)
        m_hat = np.zeros(n)
        for j in range(W):
            b, e = o.chunk_range(n, W, j)
            m_hat[b:e] = code[b:e] * F64(s_srv[j])
        u = m_hat / d.astype(F64)
        p = rng.normal(0, 0.02, n).astype(F32)
        before = p.astype(F64)
        m = np.zeros(n, F32)
        ratio = o.lamb_compressed_ratio(W, sbits, s_srv, d, p)
        want = np.linalg.norm(before) / np.linalg.norm(u)
        assert abs(F64(ratio) - want) <= 1e-6 * want, (W, n, ratio, want)
        for j in range(W):
            o.lamb_apply_chunk(j, W, LAMB_LR, ratio, sbits, s_srv[j], d, p, m)
        assert np.array_equal(m.astype(F64), m_hat)
        delta = p.astype(F64) - before
        np.testing.assert_allclose(delta, -lr * F64(ratio) * u, rtol=1e-4,
                                   atol=4 * float(np.max(ulp(p))))
        assert abs(np.linalg.norm(delta) - lr * np.linalg.norm(before)) <= 1e-5 * lr * np.linalg.norm(before)
        # p = 0: ratio 1, the 1-bit Adam update
        z, za = np.zeros(n, F32), np.zeros(n, F32)
        assert o.lamb_compressed_ratio(W, sbits, s_srv, d, z) == 1.0
        for j in range(W):
            o.lamb_apply_chunk(j, W, LAMB_LR, F32(1.0), sbits, s_srv[j], d, z, m)
        o.apply_update(LAMB_LR, sbits, s_srv, d, za, m)
        assert np.array_equal(z.view(np.uint32), za.view(np.uint32))


def pin_lamb_brute_force_message_passing(o, seed=24):
    """Whole compressed 1-bit LAMB steps against the float64 message-passing
    brute force with the LAMB update."""
    rng = np.random.default_rng(seed)
    hp = dict(HP, lr=LAMB_LR)
    for W in (1, 2, 3, 8):
        for n in (5, 33, 200, 300):
            p = rng.normal(0, 0.02, n).astype(F32)
            m = rng.normal(0, 1e-3, n).astype(F32)
            d = (np.sqrt(rng.uniform(1e-7, 1e-5, n)) + 1e-8).astype(F32)
            e_w = [rng.normal(0, 2e-4, n).astype(F32) for _ in range(W)]
            e_s = rng.normal(0, 2e-4, n).astype(F32)
            for _ in range(2):
                grads = [rng.normal(0, 1e-3, n).astype(F32) for _ in range(W)]
                ref = brute_force_step(W, m.astype(F64), d.astype(F64), p.astype(F64),
                                       [g.astype(F64) for g in grads],
                                       [e.astype(F64) for e in e_w], e_s.astype(F64), lamb=True,
                                       lr=LAMB_LR)
                bits, scales = [], []
                for w in range(W):
                    b, s = o.worker_compress(hp["beta1"], m, grads[w], e_w[w])
                    bits.append(b)
                    scales.append(s)
                sb, ss = o.server_compress(bits, np.array(scales, F32), e_s)
                ratio = o.lamb_compressed_ratio(W, sb, ss, d, p)
                assert abs(F64(ratio) - ref["ratio"]) <= 1e-5 * ref["ratio"], (W, n)
                for j in range(W):
                    o.lamb_apply_chunk(j, W, hp["lr"], ratio, sb, ss[j], d, p, m)
                np.testing.assert_allclose(m, ref["m"], rtol=1e-5, atol=1e-12)
                np.testing.assert_allclose(p, ref["p"], rtol=1e-5, atol=1e-8)


def pin_lamb_frozen_ratio_run(o, seed=25):
    """The frozen-ratio reading of 1-bit LAMB, end to end on OracleRun:
    LAMB warmup steps, then the freeze keeping the last warmup step's trust
    ratios (like the variance), then compressed steps that scale each
    tensor's update by the kept ratio.  Against float64: a LAMB warmup run
    beside it (numpy's ||p|| / ||r||, the step -lr ratio r), whose last
    ratios are the kept ones, and for each compressed step the
    message-passing brute force with those ratios from the run's state."""
    from oracle import OracleRun

    rng = np.random.default_rng(seed)
    W, sizes, Tw = 3, (200, 33, 0), 3
    hp = dict(HP, lr=LAMB_LR)
    lr = F64(F32(LAMB_LR))
    b1, b2, eps = F64(F32(HP["beta1"])), F64(F32(HP["beta2"])), F64(F32(HP["eps"]))
    params = [rng.normal(0, 0.02, n).astype(F32) for n in sizes]
    run = OracleRun(params, W, hp, oracle=o, lamb=True, lamb_frozen=True)
    P = [a.astype(F64) for a in params]
    M = [np.zeros(n) for n in sizes]
    V = [np.zeros(n) for n in sizes]
    kept = np.ones(len(sizes))
    for t in range(1, Tw + 1):
        g = [[rng.normal(0, 1e-3, n).astype(F32) for n in sizes] for _ in range(W)]
        run.warmup_step(g)
        for k, n in enumerate(sizes):
            gbar = sum(g[w][k].astype(F64) for w in range(W)) / W
            M[k] = b1 * M[k] + (1 - b1) * gbar
            V[k] = b2 * V[k] + (1 - b2) * gbar * gbar
            r = (M[k] / (1 - b1 ** t)) / (np.sqrt(V[k] / (1 - b2 ** t)) + eps)
            if n and np.linalg.norm(P[k]) > 0 and np.linalg.norm(r) > 0:
                kept[k] = np.linalg.norm(P[k]) / np.linalg.norm(r)
            else:
                kept[k] = 1.0
            P[k] = P[k] - lr * kept[k] * r
            assert abs(F64(run.ratio[k]) - kept[k]) <= 1e-5 * kept[k], (t, k)
    run.freeze()
    assert np.array_equal(run.frozen_ratio, run.ratio)
    for _ in range(3):
        g = [[rng.normal(0, 1e-3, n).astype(F32) for n in sizes] for _ in range(W)]
        before = [(run.m[k].astype(F64), run.d[k].astype(F64), run.p[k].astype(F64),
                   [run.e_w[w][k].astype(F64) for w in range(W)], run.e_s[k].astype(F64))
                  for k in range(len(sizes))]
        run.compressed_step(g)
        assert np.array_equal(run.ratio, run.frozen_ratio)   # not recomputed
        for k, n in enumerate(sizes):
            m, d, p, e_w, e_s = before[k]
            ref = brute_force_step(W, m, d, p, [g[w][k].astype(F64) for w in range(W)], e_w, e_s,
                                   lamb=True, lr=LAMB_LR, ratio=kept[k])
            np.testing.assert_allclose(run.m[k], ref["m"], rtol=1e-5, atol=1e-12)
            np.testing.assert_allclose(run.p[k], ref["p"], rtol=1e-5, atol=1e-8)


# ---------------------------------------------------------------------------
# communication volume                              [1BA, Abstract]
# ---------------------------------------------------------------------------

def read_golden(name: str) -> dict:
    """key = value lines of a fixture under tests/golden (# comments)."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = line.split("=", 1)
                out[k.strip()] = float(v)
    return out


def pin_communication_volume(o, seed=11):
    """A compressed step puts 2 (W-1) (n/8 + 4W) bytes on the wire for n a
    multiple of 32 (every chunk's words plus a 4-byte scale, worker stage
    and server stage), against 2 (W-1) 4n for the same exchange in fp32:
    32n / (n + 32W), about 32x.  Over a run whose first fraction f of the
    steps is uncompressed Adam the volume falls by 1 / (f + (1-f)/ratio);
    the pages' "up to 5x" with "typically 20%" warmup fits this."""
    rng = np.random.default_rng(seed)
    for W in (2, 4, 8):
        for n in (256, 4096, 32 * 1000):
            z = np.zeros(n)
            res = brute_force_step(W, z, np.ones(n), z, [rng.normal(size=n) for _ in range(W)],
                                   [z] * W, z)
            assert res["wire_bytes"] == 2 * (W - 1) * (n // 8 + 4 * W), (W, n)
            words = sum(o.num_words(o.chunk_range(n, W, j)[1] - o.chunk_range(n, W, j)[0])
                        for j in range(W))
            assert 4 * words == n // 8
    fig = read_golden("communication_volume.txt")
    ratio = 32.0
    at = lambda f: 1.0 / (f + (1.0 - f) / ratio)
    assert at(fig["warmup_fraction_typical"]) <= fig["volume_reduction_up_to"] <= at(0.15)


ALL_PINS = [
    pin_warmup_matches_torch_adam,
    pin_freeze_is_last_adam_denominator,
    pin_packing_matches_numpy,
    pin_exhaustive_sign_patterns,
    pin_sign_rule_and_special_values,
    pin_compressor_is_scale_times_sign,
    pin_error_feedback_telescopes,
    pin_w1_lossless_is_preconditioned_momentum_sgd,
    pin_w1_server_is_identity,
    pin_identical_workers,
    pin_chunk_layout,
    pin_brute_force_message_passing,
    pin_communication_volume,
    pin_lamb_warmup_from_zero_params_is_adam,
    pin_lamb_warmup_layerwise_step,
    pin_lamb_compressed_update,
    pin_lamb_brute_force_message_passing,
    pin_lamb_frozen_ratio_run,
]
