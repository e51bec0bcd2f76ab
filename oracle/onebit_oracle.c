/*
 * onebit_oracle.c -- CPU oracle for the compression-phase step of 1-bit Adam.
 *
 * TEST INFRASTRUCTURE ONLY.  The product library never includes, links,
 * loads or calls this file.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg use it, through oracle/__init__.py.
 *
 * Plain, slow, single-threaded C99.  It is compiled with -O2
 * -ffp-contract=off and without -ffast-math, and the file refuses to build
 * unless float expressions are evaluated in float (FLT_EVAL_METHOD == 0).
 * So each float expression statement below is one IEEE-754 binary32
 * operation, rounded to nearest-even, taken in the order written.  Sums
 * of squares for the scales are taken in double, sequentially.
 *
 * Everything here works on ONE tensor of n elements, stored densely (no
 * padding).  A list of tensors is a list of independent problems: scales,
 * sign packing and server chunks are all per tensor.
 *
 * What it follows.  The method is stated in prose on the review page
 * "1-bit Adam: Communication Efficient Large-Scale Training with Adam's
 * Convergence Speed" (cited below as [1BA]):
 *   [1BA, Abstract]            1-bit compression with error compensation;
 *                              Adam's variance becomes stable after a
 *                              warmup and is then used as a fixed
 *                              preconditioner.
 *   [1BA, Proposed method, 1]  a full-precision Adam warmup (about 20% of
 *                              the steps), then 1-bit compressed momentum
 *                              SGD for the rest.
 *   [1BA, Proposed method, 2]  the variance serves as the preconditioner of
 *                              that momentum SGD.
 *   [1BA, Proposed method, 3]  the error-compensated compression is applied
 *                              to the momentum, not to the gradient.
 *   [1BA, Proposed method, 4]  a custom collective carries the compressed
 *                              momentum between workers.
 * The pages print no equations.  The readings taken here (the scale is the
 * RMS of the tensor, sign(0) = +1, a worker stage and a server stage each
 * with its own error feedback, per-chunk server scales, the bias-corrected
 * variance as the frozen preconditioner, and the averaged momentum
 * replacing every worker's momentum) are listed with their reasons in the
 * design notes of this repository.
 *
 * Pins: every function here is checked against something other than
 * itself by tests/test_oracle_pins.py (textbook Adam and momentum SGD from
 * torch.optim, numpy's bit packing and norms, exhaustive patterns,
 * telescoping of the error feedback, a message-passing brute force).
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#if !defined(FLT_EVAL_METHOD) || FLT_EVAL_METHOD != 0
#error "the oracle needs float expressions evaluated in float (FLT_EVAL_METHOD == 0)"
#endif

#define ORC_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------ */
/* Small helpers                                                       */
/* ------------------------------------------------------------------ */

/* Number of 32-bit sign words of a tensor of n elements. */
ORC_API int64_t orc_num_words(int64_t n) { return (n + 31) / 32; }

/* The 1-bit code of x: 1 means +1, 0 means -1.  sign(0) = +1, so both
 * +0.0 and -0.0 give 1 (x >= 0 holds for -0.0); NaN gives 0. */
static int sign_bit(float x) { return x >= 0.0f ? 1 : 0; }

/* sigma * s for a code bit; exact (only the sign of s changes). */
static float signed_scale(int bit, float s) { return bit ? s : -s; }

/* Bit i of a packed array: bit (i mod 32) of word (i div 32). */
static int get_bit(const uint32_t *words, int64_t i) {
    return (int)((words[i >> 5] >> (i & 31)) & 1u);
}

/* Pack the codes of x[0..n) 32 per word, bit k of word i = element 32i+k.
 * Bits past n in the last word are 0. */
static void pack_signs(int64_t n, const float *x, uint32_t *words) {
    memset(words, 0, (size_t)orc_num_words(n) * sizeof(uint32_t));
    for (int64_t i = 0; i < n; ++i)
        if (sign_bit(x[i])) words[i >> 5] |= (uint32_t)1u << (i & 31);
}

/* Scale of the 1-bit compressor: RMS of the values, s = ||x||_2 / sqrt(n),
 * from a sequential double sum of squares, rounded once to float.  An
 * empty range has scale 0. */
static float rms_scale(double sum_sq, int64_t count) {
    if (count <= 0) return 0.0f;
    return (float)sqrt(sum_sq / (double)count);
}

/* ------------------------------------------------------------------ */
/* Server chunks of the two-stage compressed allreduce                 */
/* ------------------------------------------------------------------ */

/* [1BA, Proposed method, 4]: the compressed momentum of a tensor is split
 * among W servers.  With nw = ceil(n/32) sign words, each server owns a
 * contiguous run of cw = roundup(ceil(nw/W), 4) words; server j owns words
 * [j*cw, min(nw, (j+1)*cw)), that is elements
 * [min(n, 32*j*cw), min(n, 32*(j+1)*cw)).  Trailing servers may own
 * nothing. */
ORC_API void orc_chunk_range(int64_t n, int W, int j, int64_t *begin, int64_t *end) {
    const int64_t nw = orc_num_words(n);
    const int64_t per = (nw + W - 1) / W;
    const int64_t cw = ((per + 3) / 4) * 4;
    int64_t wb = (int64_t)j * cw;
    int64_t we = wb + cw;
    if (wb > nw) wb = nw;
    if (we > nw) we = nw;
    int64_t b = 32 * wb;
    int64_t e = 32 * we;
    if (b > n) b = n;
    if (e > n) e = n;
    *begin = b;
    *end = e;
}

/* ------------------------------------------------------------------ */
/* Warmup phase: full-precision Adam                                   */
/* ------------------------------------------------------------------ */

/* [1BA, Proposed method, 1]: the warmup is plain Adam on the averaged
 * gradient.  For element i of one step t (t = 1, 2, ...) over W workers'
 * gradients g[w]:
 *   gbar = (g_0 + g_1 + ... + g_{W-1}) / W   (sum from +0.0, in w order)
 *   m = beta1*m + (1-beta1)*gbar
 *   v = beta2*v + (1-beta2)*gbar^2
 * updated in place, and the returned direction of the step
 *   r = (m/bc1) / (sqrt(v/bc2) + eps),
 * with bc1 = 1 - beta1^t and bc2 = 1 - beta2^t taken in double and rounded
 * once to float by the caller. */
static float adam_moments_and_direction(int64_t i, int W, const float *const *g, float beta1,
                                        float beta2, float bc1, float bc2, float eps, float *m,
                                        float *v) {
    const float c1 = 1.0f - beta1;
    const float c2 = 1.0f - beta2;
    const float wf = (float)W;
    float acc = 0.0f;
    for (int w = 0; w < W; ++w) acc = acc + g[w][i];
    const float gbar = acc / wf;

    const float m_old = beta1 * m[i];
    const float m_new = c1 * gbar;
    m[i] = m_old + m_new;

    const float gsq = gbar * gbar;
    const float v_old = beta2 * v[i];
    const float v_new = c2 * gsq;
    v[i] = v_old + v_new;

    const float mhat = m[i] / bc1;
    const float vhat = v[i] / bc2;
    const float root = sqrtf(vhat);
    const float denom = root + eps;
    return mhat / denom;
}

/* One Adam warmup step: the moments and direction above, then
 *   p = p - lr * r. */
ORC_API void orc_adam_warmup_step(int64_t n, int W, int t, float beta1, float beta2, float eps,
                                  float lr, const float *const *g, float *m, float *v, float *p) {
    const float bc1 = (float)(1.0 - pow((double)beta1, (double)t));
    const float bc2 = (float)(1.0 - pow((double)beta2, (double)t));
    for (int64_t i = 0; i < n; ++i) {
        const float ratio = adam_moments_and_direction(i, W, g, beta1, beta2, bc1, bc2, eps, m, v);
        const float delta = lr * ratio;
        p[i] = p[i] - delta;
    }
}

/* [1BA, Abstract; Proposed method, 2]: after Tw warmup steps the variance
 * is frozen.  The preconditioner kept for the compression phase is the
 * denominator Adam used at its last warmup step:
 *   d = sqrt(v / bc2(Tw)) + eps. */
ORC_API void orc_freeze(int64_t n, int Tw, float beta2, float eps, const float *v, float *d) {
    const float bc2 = (float)(1.0 - pow((double)beta2, (double)Tw));
    for (int64_t i = 0; i < n; ++i) {
        const float vhat = v[i] / bc2;
        const float root = sqrtf(vhat);
        d[i] = root + eps;
    }
}

/* ------------------------------------------------------------------ */
/* Compression phase                                                   */
/* ------------------------------------------------------------------ */

/* Worker stage for one worker [1BA, Proposed method, 3; Abstract]:
 *   m_w = beta1*m + (1-beta1)*g_w        (this worker's momentum)
 *   x   = m_w + e_w                      (add the worker's error)
 *   s   = ||x||_2 / sqrt(n)              (scale, double sum, one rounding)
 *   bits: 1 where x >= 0                 (32 per word)
 *   e_w = x - sign(x)*s                  (new error feedback)
 * e is updated in place.  bits receives ceil(n/32) words.  x_out, if not
 * NULL, receives x.  Returns 0, or -1 when out of memory. */
ORC_API int orc_worker_compress(int64_t n, float beta1, const float *m, const float *g,
                                float *e, uint32_t *bits, float *x_out, float *scale_out) {
    const float c1 = 1.0f - beta1;
    float *x = x_out;
    if (!x) {
        x = (float *)calloc((size_t)(n > 0 ? n : 1), sizeof(float));
        if (!x) return -1;
    }
    double sum_sq = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        const float m_old = beta1 * m[i];
        const float m_new = c1 * g[i];
        const float m_w = m_old + m_new;
        x[i] = m_w + e[i];
        sum_sq += (double)x[i] * (double)x[i];
    }
    const float s = rms_scale(sum_sq, n);
    pack_signs(n, x, bits);
    for (int64_t i = 0; i < n; ++i) e[i] = x[i] - signed_scale(sign_bit(x[i]), s);
    *scale_out = s;
    if (x != x_out) free(x);
    return 0;
}

/* Server stage of one chunk [1BA, Proposed method, 3-4]: server j receives
 * chunk j of every worker's packed signs plus every worker's scale.  For
 * element i of chunk j:
 *   acc = +0.0; acc = acc + sign_w(i)*s_w  for w = 0..W-1 in order
 *   y   = acc / W + e_s(i)               (average, plus the server error)
 * then the chunk is compressed again:
 *   s'_j = ||y over chunk j||_2 / sqrt(len_j)   (0 for an empty chunk)
 *   sbits: 1 where y >= 0
 *   e_s = y - sign(y)*s'_j.
 * bits[w] holds worker w's ceil(n/32) words, s[w] its scale.  Only chunk
 * j's elements of e_s and y_out (if not NULL) and chunk j's words of sbits
 * are written (chunks start on 128-element boundaries, so no word is
 * shared with another chunk).  *s_srv_j receives s'_j.  Returns 0 or -1. */
ORC_API int orc_server_compress_chunk(int64_t n, int W, int j, const uint32_t *const *bits,
                                      const float *s, float *e_s, uint32_t *sbits, float *s_srv_j,
                                      float *y_out) {
    const float wf = (float)W;
    int64_t b, e;
    orc_chunk_range(n, W, j, &b, &e);
    /* y of element i is y[i - b]: the chunk's own values, either in y_out
     * (whose element i is y_out[i]) or in a buffer of the chunk's length */
    float *y = y_out ? y_out + b : (float *)calloc((size_t)(e > b ? e - b : 1), sizeof(float));
    if (!y) return -1;
    double sum_sq = 0.0;
    for (int64_t i = b; i < e; ++i) {
        float acc = 0.0f;
        for (int w = 0; w < W; ++w) acc = acc + signed_scale(get_bit(bits[w], i), s[w]);
        const float avg = acc / wf;
        y[i - b] = avg + e_s[i];
        sum_sq += (double)y[i - b] * (double)y[i - b];
    }
    const float sj = rms_scale(sum_sq, e - b);
    if (e > b)  /* an empty chunk owns no word, not even the tensor's last */
        for (int64_t k = b / 32; k < (e + 31) / 32; ++k) sbits[k] = 0u;
    for (int64_t i = b; i < e; ++i)
        if (sign_bit(y[i - b])) sbits[i >> 5] |= (uint32_t)1u << (i & 31);
    for (int64_t i = b; i < e; ++i) e_s[i] = y[i - b] - signed_scale(sign_bit(y[i - b]), sj);
    *s_srv_j = sj;
    if (!y_out) free(y);
    return 0;
}

/* Server stage of a whole tensor: every chunk j = 0..W-1 as above.  sbits
 * receives ceil(n/32) words, s_srv the W chunk scales, y_out (if not
 * NULL) y.  Returns 0 or -1. */
ORC_API int orc_server_compress(int64_t n, int W, const uint32_t *const *bits, const float *s,
                                float *e_s, uint32_t *sbits, float *s_srv, float *y_out) {
    memset(sbits, 0, (size_t)orc_num_words(n) * sizeof(uint32_t));
    for (int j = 0; j < W; ++j)
        if (orc_server_compress_chunk(n, W, j, bits, s, e_s, sbits, &s_srv[j], y_out) != 0)
            return -1;
    return 0;
}

/* Gather and update of one chunk [1BA, Proposed method, 1-2]: every worker
 * receives all server chunks and decodes the averaged momentum
 * m_hat = sign'(i)*s'_j (exact), which replaces the momentum; the
 * parameters take one momentum SGD step preconditioned by the frozen
 * denominator d:
 *   p = p - lr * (m_hat / d);   m = m_hat.
 * Only chunk j's elements are written. */
ORC_API void orc_apply_chunk(int64_t n, int W, int j, float lr, const uint32_t *sbits,
                             float s_srv_j, const float *d, float *p, float *m) {
    int64_t b, e;
    orc_chunk_range(n, W, j, &b, &e);
    for (int64_t i = b; i < e; ++i) {
        const float m_hat = signed_scale(get_bit(sbits, i), s_srv_j);
        const float ratio = m_hat / d[i];
        const float delta = lr * ratio;
        p[i] = p[i] - delta;
        m[i] = m_hat;
    }
}

/* Gather and update of a whole tensor: every chunk as above. */
ORC_API void orc_apply(int64_t n, int W, float lr, const uint32_t *sbits, const float *s_srv,
                       const float *d, float *p, float *m) {
    for (int j = 0; j < W; ++j) orc_apply_chunk(n, W, j, lr, sbits, s_srv[j], d, p, m);
}

/* ------------------------------------------------------------------ */
/* 1-bit LAMB: layerwise adaptive learning rates                       */
/* ------------------------------------------------------------------ */

/* The review page "1-bit LAMB: Communication Efficient Large-Scale
 * Large-Batch Training with LAMB's Convergence Speed" gives only its
 * abstract: LAMB's adaptive layerwise learning rates are kept while the
 * communication is compressed, on top of the 1-bit Adam scheme above.  It
 * prints no update rule.  The reading taken here is the plainest the
 * abstract supports:
 *   - the layerwise rate is LAMB's trust ratio of each tensor,
 *       ratio = ||p|| / ||u||   (1 when either norm is 0),
 *     u being the tensor's update direction, and the step is
 *       p = p - (lr * ratio) * u;
 *   - during the warmup u is full-precision Adam's m_hat / (sqrt(v_hat) +
 *     eps) (warmup = LAMB);
 *   - during the compression phase u = m_hat / d, m_hat being the momentum
 *     decoded from the compressed collective and d the frozen denominator:
 *     every worker holds the same p and m_hat after the gather, so every
 *     worker computes the same ratio although the momentum was compressed;
 *   - the ratio is recomputed at every step (nothing else is frozen).
 * Norms are sums of squares in double (sequential), the ratio
 * (float)sqrt(P / U), rounded once; lr * ratio is one float
 * multiplication.  With ratio = 1 the steps are exactly the Adam warmup and
 * the 1-bit Adam update above. */

/* Sum of squares in double, sequential. */
ORC_API double orc_sum_squares(int64_t n, const float *x) {
    double s = 0.0;
    for (int64_t i = 0; i < n; ++i) s += (double)x[i] * (double)x[i];
    return s;
}

/* LAMB's trust ratio from the squared norms of p and of the update u. */
static float trust_ratio(double p_sq, double u_sq) {
    if (p_sq > 0.0 && u_sq > 0.0) return (float)sqrt(p_sq / u_sq);
    return 1.0f;
}

/* One warmup step of 1-bit LAMB: the Adam moments of the averaged
 * gradient as in orc_adam_warmup_step, then the tensor's trust ratio of
 * p (before the step) and the Adam direction r, then the step.  *ratio_out
 * receives the ratio.  Returns 0, or -1 when out of memory. */
ORC_API int orc_lamb_warmup_step(int64_t n, int W, int t, float beta1, float beta2, float eps,
                                 float lr, const float *const *g, float *m, float *v, float *p,
                                 float *ratio_out) {
    const float bc1 = (float)(1.0 - pow((double)beta1, (double)t));
    const float bc2 = (float)(1.0 - pow((double)beta2, (double)t));
    float *r = (float *)calloc((size_t)(n > 0 ? n : 1), sizeof(float));
    if (!r) return -1;
    for (int64_t i = 0; i < n; ++i)
        r[i] = adam_moments_and_direction(i, W, g, beta1, beta2, bc1, bc2, eps, m, v);
    const float ratio = trust_ratio(orc_sum_squares(n, p), orc_sum_squares(n, r));
    const float lr_t = lr * ratio;
    for (int64_t i = 0; i < n; ++i) {
        const float delta = lr_t * r[i];
        p[i] = p[i] - delta;
    }
    free(r);
    *ratio_out = ratio;
    return 0;
}

/* The compression phase's trust ratio of one tensor, once every server
 * chunk's words and scale are known: p before the step, and the direction
 * u = m_hat / d with m_hat = sign'(i) * s'_j decoded from the server words.
 * ||u||^2 is taken as the sum of (m_hat / d)^2 over the elements, each
 * quotient formed in double from the float values. */
ORC_API float orc_lamb_compressed_ratio(int64_t n, int W, const uint32_t *sbits, const float *s_srv,
                                        const float *d, const float *p) {
    double u_sq = 0.0;
    for (int j = 0; j < W; ++j) {
        int64_t b, e;
        orc_chunk_range(n, W, j, &b, &e);
        for (int64_t i = b; i < e; ++i) {
            const double q = (double)signed_scale(get_bit(sbits, i), s_srv[j]) / (double)d[i];
            u_sq += q * q;
        }
    }
    return trust_ratio(orc_sum_squares(n, p), u_sq);
}

/* Gather and update of one chunk of the compression phase of 1-bit LAMB:
 * the 1-bit Adam update of orc_apply_chunk with the tensor's layerwise
 * rate lr * ratio in place of lr:
 *   p = p - (lr * ratio) * (m_hat / d);   m = m_hat. */
ORC_API void orc_lamb_apply_chunk(int64_t n, int W, int j, float lr, float ratio,
                                  const uint32_t *sbits, float s_srv_j, const float *d, float *p,
                                  float *m) {
    const float lr_t = lr * ratio;
    orc_apply_chunk(n, W, j, lr_t, sbits, s_srv_j, d, p, m);
}
