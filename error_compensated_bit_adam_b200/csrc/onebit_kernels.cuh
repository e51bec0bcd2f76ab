// onebit_kernels.cuh -- device code of libonebit (sm_100a).
//
// The compression-phase step of 1-bit Adam ("1-bit Adam: Communication
// Efficient Large-Scale Training with Adam's Convergence Speed", review
// page, sections "Abstract" and "Proposed method") as five HBM-streaming
// kernels over a list of 4096-element tiles:
//
//   ob_pack_kernel          worker stage, all W workers of a tile per CTA
//   ob_scale_kernel         worker scales per (tensor, worker)
//   ob_server_kernel        server stage of a tile
//   ob_scale_kernel         server scales per (tensor, chunk)
//   ob_apply_kernel         gather, decode, preconditioned update
//
// plus the warmup Adam step, the freeze and an error decoder used when the
// host reads state.  No step is a dense contraction, so no tensor cores:
// every kernel is a stream of coalesced 16-byte loads and stores, bound by
// HBM bandwidth.
//
// Numerics.  Every fp32 operation is written with an explicit
// round-to-nearest intrinsic (__fmul_rn, __fadd_rn, __fsub_rn, __fdiv_rn,
// __fsqrt_rn), so nvcc cannot contract a*b+c into an FMA, and the order of
// operations is the method's: the results are the same IEEE binary32
// values a plain sequential CPU evaluation gives.  Sums of squares for the
// scales are taken in fp64 in a fixed order (per thread, warp butterfly,
// warps in order, tiles in order), so results repeat run to run.
//
// Lazy error buffers.  e_w = x - sign(x) s_w needs s_w, which needs all of
// x.  Rather than a second pass over x, the worker error is stored as the
// pair (x, s_w) and decoded where it is next used:
//   e_w = fl(x - sign(x) s_w)   -- the same rounding an eager pass would do.
// The server error is stored the same way as (y, s'_j).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/onebit.h"

namespace onebit {

constexpr int kThreads = 256;              // threads per CTA of the tile kernels
constexpr int kWarps = kThreads / 32;
constexpr int kUnroll = 4;                 // float4 slots per thread per tile
constexpr int kTile = kThreads * 4 * kUnroll;  // 4096 elements per tile
constexpr int kScaleThreads = 256;         // threads of the scale kernels
constexpr int kPackStages = 2;             // workers in flight in the worker-stage pipeline
constexpr int kPackSmemBytes = kPackStages * 2 * kUnroll * kThreads * 16;  // 64 KiB: 3 CTAs per SM
constexpr unsigned kFull = 0xffffffffu;

// One unit of work: up to kTile consecutive elements of one tensor that all
// belong to one server chunk.  begin is the padded-layout element offset of
// the tile's first element (a multiple of 128); count is the number of real
// (non-padding) elements.
struct Tile {
    int64_t begin;
    int32_t count;
    int32_t tensor;
    int32_t chunk;
    int32_t reserved;
};
static_assert(sizeof(Tile) == 24, "Tile layout");
static_assert(kWarps * kUnroll * 128 == kTile, "warp spans cover a tile");
static_assert(kUnroll * 4 <= 32, "a warp's sign words fit one store");

// ---------------------------------------------------------------- helpers

__device__ __forceinline__ float signed_scale(bool plus, float s) { return plus ? s : -s; }

// The 1-bit code: +1 for x >= 0 (so +0.0 and -0.0 give +1), else -1.
__device__ __forceinline__ bool code_of(float x) { return x >= 0.0f; }

// Error feedback stored lazily as (x, s): e = fl(x - sign(x) s).
__device__ __forceinline__ float decode_error(float x, float s) {
    return __fsub_rn(x, signed_scale(code_of(x), s));
}

// +-s as a float, from a sign word: bit b of `word` set -> +s, clear -> -s.
// s >= 0, so only the sign bit changes: (~word << (31 - b)) keeps the
// inverted bit in bit 31.
__device__ __forceinline__ float signed_from_bit(uint32_t word, int b, uint32_t s_bits) {
    return __uint_as_float(((~word << (31 - b)) & 0x80000000u) | s_bits);
}

__device__ __forceinline__ float get(const float4 &v, int k) {
    return k == 0 ? v.x : (k == 1 ? v.y : (k == 2 ? v.z : v.w));
}
__device__ __forceinline__ void set(float4 &v, int k, float f) {
    if (k == 0) v.x = f; else if (k == 1) v.y = f; else if (k == 2) v.z = f; else v.w = f;
}

// Streaming 16-byte accesses: every byte is touched once per step, so the
// lines are marked evict-first (.cs), keeping L2 for the packed words and
// scales.  The load is a plain (non-volatile, no memory clobber) asm, so the
// compiler may issue a thread's later loads before its earlier stores; that
// is correct because no kernel here loads an address after the same thread
// stored to it (each element is read, then written once, the store
// depending on the load).
__device__ __forceinline__ float4 ld_stream(const float *p) {
    float4 v;
    asm("ld.global.cs.v4.f32 {%0, %1, %2, %3}, [%4];"
        : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
        : "l"(p));
    return v;
}
__device__ __forceinline__ void st_stream(float *p, const float4 &v) {
    asm volatile("st.global.cs.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z),
                 "f"(v.w));
}

// Asynchronous 16-byte global -> shared copies (sm_80+ LDGSTS), with an L2
// evict-first policy: the CTA queues the next workers' inputs while it
// computes on the current one.  Completion is awaited per thread with
// cp.async.wait_group (a hardware wait, no polling).
__device__ __forceinline__ uint64_t evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, uint64_t pol) {
    const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem),
                 "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// OR together the 4-bit groups of the 8 lanes that share one 32-bit sign
// word.  Lane l holds elements 4l..4l+3 of the warp's 128-element slot, so
// its nibble goes to bits 4*(l%8)..4*(l%8)+3 of word l/8.  Every lane of
// the group ends with the whole word.
__device__ __forceinline__ uint32_t gather_word(uint32_t nibble, int lane) {
    uint32_t v = nibble << (4 * (lane & 7));
    v |= __shfl_xor_sync(kFull, v, 1);
    v |= __shfl_xor_sync(kFull, v, 2);
    v |= __shfl_xor_sync(kFull, v, 4);
    return v;
}

// Element offset, within a tile, of slot u of a thread when each warp owns a
// contiguous span of kUnroll * 128 elements: warp `warp`'s slot u covers
// [512 warp + 128 u, +128), lane l holding elements 4l..4l+3 of it.  The
// warp's sign words for the span are then 4 * kUnroll consecutive words.
__device__ __forceinline__ int span_off(int warp, int lane, int u) {
    return (kUnroll * 128) * warp + 128 * u + 4 * lane;
}

// After gather_word for every slot, lanes 0, 8, 16, 24 hold words 4u..4u+3
// of slot u.  Bring word L of the warp's 4 * kUnroll to lane L so the warp
// stores all of them with one 64-byte, sector-aligned write.
__device__ __forceinline__ uint32_t collect_words(const uint32_t (&word)[kUnroll], int lane) {
    uint32_t mine = 0;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const uint32_t v = __shfl_sync(kFull, word[u], 8 * (lane & 3));
        if ((lane >> 2) == u) mine = v;
    }
    return mine;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}

// Fixed-order fp64 sum over a CTA of kScaleThreads threads (result valid in
// thread 0).
__device__ __forceinline__ double block_sum(double v, double *smem) {
    v = warp_sum(v);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) smem[warp] = v;
    __syncthreads();
    double acc = 0.0;
    if (threadIdx.x == 0)
        for (int k = 0; k < kScaleThreads / 32; ++k) acc += smem[k];
    return acc;
}

// Real elements (0..4) of the float4 slot at tile offset off.
__device__ __forceinline__ int slot_real(int count, int off) { return min(4, max(0, count - off)); }

// ------------------------------------------------------------ warmup Adam

struct WarmupParams {
    const Tile *tiles;
    const float *g[OB_MAX_WORKERS];  // worker gradients, padded layout
    float *m, *v, *p;
    int W;
    float beta1, beta2, c1, c2, bc1, bc2, eps, lr;
};

// [1BA, Proposed method, 1]: one full-precision Adam step on the averaged
// gradient, elementwise.
__global__ void __launch_bounds__(kThreads) ob_warmup_kernel(const __grid_constant__ WarmupParams P) {
    const Tile tile = P.tiles[blockIdx.x];
    const float wf = (float)P.W;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int off = 4 * ((int)threadIdx.x + kThreads * u);
        const int real = slot_real(tile.count, off);
        if (real == 0) continue;
        const int64_t i = tile.begin + off;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int w = 0; w < P.W; ++w) {
            const float4 g = ld_stream(P.g[w] + i);
            acc.x = __fadd_rn(acc.x, g.x);
            acc.y = __fadd_rn(acc.y, g.y);
            acc.z = __fadd_rn(acc.z, g.z);
            acc.w = __fadd_rn(acc.w, g.w);
        }
        float4 m = ld_stream(P.m + i), v = ld_stream(P.v + i), p = ld_stream(P.p + i);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (k >= real) break;  // padding keeps its values
            const float gbar = __fdiv_rn(get(acc, k), wf);
            const float mk = __fadd_rn(__fmul_rn(P.beta1, get(m, k)), __fmul_rn(P.c1, gbar));
            const float vk = __fadd_rn(__fmul_rn(P.beta2, get(v, k)),
                                       __fmul_rn(P.c2, __fmul_rn(gbar, gbar)));
            const float mhat = __fdiv_rn(mk, P.bc1);
            const float vhat = __fdiv_rn(vk, P.bc2);
            const float denom = __fadd_rn(__fsqrt_rn(vhat), P.eps);
            const float delta = __fmul_rn(P.lr, __fdiv_rn(mhat, denom));
            set(m, k, mk);
            set(v, k, vk);
            set(p, k, __fsub_rn(get(p, k), delta));
        }
        st_stream(P.m + i, m);
        st_stream(P.v + i, v);
        st_stream(P.p + i, p);
    }
}

// ----------------------------------------------------------------- freeze

// [1BA, Abstract; Proposed method, 2]: d = sqrt(v / bc2) + eps, in place.
__global__ void __launch_bounds__(kThreads) ob_freeze_kernel(const Tile *tiles, float *v, float bc2,
                                                             float eps) {
    const Tile tile = tiles[blockIdx.x];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int off = 4 * ((int)threadIdx.x + kThreads * u);
        const int real = slot_real(tile.count, off);
        if (real == 0) continue;
        float4 x = ld_stream(v + tile.begin + off);
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (k < real) set(x, k, __fadd_rn(__fsqrt_rn(__fdiv_rn(get(x, k), bc2)), eps));
        st_stream(v + tile.begin + off, x);
    }
}

// ----------------------------------------------------------- worker stage

struct PackParams {
    const Tile *tiles;
    int tile_base;                   // tile of blockIdx.x == 0
    int n_tiles;                     // total tiles (row length of partial)
    const float *m;                  // [n_pad] dense momentum (when m_dense)
    const uint32_t *m_bits;          // [n_pad/32] last step's server signs (when !m_dense)
    const float *m_scale;            // [T][W] last step's server scales (when !m_dense)
    int m_dense;
    const float *g[OB_MAX_WORKERS];  // element i of worker w at g[w][i - g_offset]
    int64_t g_offset;
    float *x;                        // [W][n_pad]: in x_prev (lazy e_w), out x
    uint32_t *bits;                  // [W][n_pad/32]
    const float *s_prev;             // [W][T]: scale that decodes x_prev
    double *partial;                 // [W][n_tiles]: sum of x^2 per tile
    int64_t n_pad;
    int W, T;
    float beta1, c1;
};

// [1BA, Proposed method, 3; Abstract]: for every worker w of one tile,
//   m_w = beta1 m + (1-beta1) g_w,  x = m_w + e_w (e_w decoded from the
//   stored (x_prev, s_prev)), sign bits of x, partial sum of x^2.
// x overwrites x_prev: with this step's scale it encodes the new e_w.
// m stays in registers across the W workers, so it is read once.  After a
// compressed step m is exactly last step's decoded server momentum
// sign' s'_j, so it is rebuilt from the server words (1/8 byte per
// parameter) instead of read as fp32 (4 bytes).
__global__ void __launch_bounds__(kThreads) ob_pack_kernel(const __grid_constant__ PackParams P) {
    const int tile_id = P.tile_base + (int)blockIdx.x;
    const Tile tile = P.tiles[tile_id];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ double red[kWarps][OB_MAX_WORKERS];

    float4 mv[kUnroll];
    int real[kUnroll];
    if (P.m_dense) {
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int off = span_off(warp, lane, u);
            real[u] = slot_real(tile.count, off);
            mv[u] = real[u] > 0 ? ld_stream(P.m + tile.begin + off) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    } else {
        const uint32_t sb = __float_as_uint(P.m_scale[tile.tensor * P.W + tile.chunk]);
        const int shift = 4 * (lane & 7);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int off = span_off(warp, lane, u);
            real[u] = slot_real(tile.count, off);
            mv[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (real[u] > 0) {
                const uint32_t word = __ldg(P.m_bits + ((tile.begin + off) >> 5));
#pragma unroll
                for (int k = 0; k < 4; ++k) set(mv[u], k, signed_from_bit(word, shift + k, sb));
            }
        }
    }
    const int64_t words_per_worker = P.n_pad >> 5;
    // Pipeline over the workers: the gradient and x_prev slots of worker
    // w + kPackStages - 1 are copied into shared memory (cp.async) while
    // worker w is computed, so HBM stays busy whatever the arithmetic's
    // latency.  Each thread reads back only the slots it copied itself, so
    // its own wait_group is the only synchronisation needed.
    extern __shared__ float4 pipe[];  // [kPackStages][2 (g, x_prev)][kUnroll][kThreads]
    const uint64_t pol = evict_first_policy();
    auto issue = [&](int w) {
        if (w < P.W) {
            const int st = w % kPackStages;
            const float *gw = P.g[w] + (tile.begin - P.g_offset);
            const float *xw = P.x + (int64_t)w * P.n_pad + tile.begin;
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                if (real[u] > 0) {
                    const int off = span_off(warp, lane, u);
                    cp_async16(&pipe[((st * 2 + 0) * kUnroll + u) * kThreads + tid], gw + off, pol);
                    cp_async16(&pipe[((st * 2 + 1) * kUnroll + u) * kThreads + tid], xw + off, pol);
                }
            }
        }
        cp_async_commit();  // one group per worker, empty past the last
    };
#pragma unroll
    for (int k = 0; k < kPackStages - 1; ++k) issue(k);
    for (int w = 0; w < P.W; ++w) {
        issue(w + kPackStages - 1);
        cp_async_wait<kPackStages - 1>();  // worker w's group has landed
        const int st = w % kPackStages;
        const float s_prev = P.s_prev[w * P.T + tile.tensor];
        float *xw = P.x + (int64_t)w * P.n_pad + tile.begin;
        uint32_t *bw = P.bits + (int64_t)w * words_per_worker + (tile.begin >> 5);
        double ss[kUnroll];
        uint32_t words[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int off = span_off(warp, lane, u);
            ss[u] = 0.0;
            uint32_t nibble = 0;
            if (real[u] > 0) {
                const float4 g = pipe[((st * 2 + 0) * kUnroll + u) * kThreads + tid];
                const float4 xp = pipe[((st * 2 + 1) * kUnroll + u) * kThreads + tid];
                float4 xo = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    if (k < real[u]) {
                        const float m_w = __fadd_rn(__fmul_rn(P.beta1, get(mv[u], k)),
                                                    __fmul_rn(P.c1, get(g, k)));
                        const float x = __fadd_rn(m_w, decode_error(get(xp, k), s_prev));
                        ss[u] = __fma_rn((double)x, (double)x, ss[u]);
                        nibble |= (uint32_t)code_of(x) << k;
                        set(xo, k, x);
                    }
                }
                st_stream(xw + off, xo);
            }
            words[u] = gather_word(nibble, lane);
        }
        const uint32_t mine = collect_words(words, lane);
        if (lane < 4 * kUnroll && (kUnroll * 128) * warp + 32 * lane < tile.count)
            bw[4 * kUnroll * warp + lane] = mine;
        double t = 0.0;
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) t += ss[u];
        t = warp_sum(t);
        if (lane == 0) red[warp][w] = t;
    }
    __syncthreads();
    if (tid < P.W) {
        double acc = 0.0;
#pragma unroll
        for (int k = 0; k < kWarps; ++k) acc += red[k][tid];
        P.partial[(int64_t)tid * P.n_tiles + tile_id] = acc;
    }
}

// ------------------------------------------------------------- scales
//
// A scale is sqrt(S / count) with S the sum of the per-tile partial sums of
// one range of tiles (a tensor for the worker scales, a server chunk for
// the server scales).  A range is cut into segments of kScaleSegTiles
// tiles; one CTA sums one segment, and the CTA that finishes last for the
// range sums the segment results in segment order.  The order of every
// addition is fixed by the layout, so the scales repeat run to run.  The
// last CTA is found with a per-range counter (thread fence, then atomic
// increment; it resets the counter), so nothing ever waits.

constexpr int kScaleSegTiles = 2048;

__device__ __forceinline__ double segment_sum(const double *v, int lo, int hi, double *smem) {
    double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
    int k = lo + (int)threadIdx.x;
    for (; k + 3 * kScaleThreads < hi; k += 4 * kScaleThreads) {
        a0 += __ldcg(v + k);
        a1 += __ldcg(v + k + kScaleThreads);
        a2 += __ldcg(v + k + 2 * kScaleThreads);
        a3 += __ldcg(v + k + 3 * kScaleThreads);
    }
    for (; k < hi; k += kScaleThreads) a0 += __ldcg(v + k);
    return block_sum((a0 + a1) + (a2 + a3), smem);
}

// One segment of range r; returns (in thread 0, with *done = true) the
// range's total when this CTA is the last of the range's nseg CTAs.
__device__ __forceinline__ bool range_sum(const double *v, int lo, int hi, int seg, int nseg,
                                          double *seg_out, unsigned *counter, double *total) {
    __shared__ double smem[kScaleThreads / 32];
    __shared__ bool last;
    const int a = lo + seg * kScaleSegTiles;
    const int b = min(hi, a + kScaleSegTiles);
    const double part = segment_sum(v, a, b, smem);
    if (nseg == 1) {
        *total = part;
        return true;
    }
    if (threadIdx.x == 0) {
        seg_out[seg] = part;
        __threadfence();
        last = atomicAdd(counter, 1u) == (unsigned)(nseg - 1);
    }
    __syncthreads();
    if (!last) return false;
    if (threadIdx.x == 0) {
        __threadfence();
        double acc = 0.0;
        for (int k = 0; k < nseg; ++k) acc += __ldcg(seg_out + k);
        *counter = 0u;
        *total = acc;
    }
    return true;
}

__device__ __forceinline__ int num_segments(int tiles) {
    return tiles <= kScaleSegTiles ? 1 : (tiles + kScaleSegTiles - 1) / kScaleSegTiles;
}

__device__ __forceinline__ float rms(double sum_sq, int64_t count) {
    return count > 0 ? __double2float_rn(__dsqrt_rn(__ddiv_rn(sum_sq, (double)count))) : 0.0f;
}

struct ScaleParams {
    const double *partial;     // per-tile sums
    int n_tiles;               // row length of partial (worker scales: one row per worker)
    const int *range_begin;    // [R+1] tile ranges
    const int *seg_base;       // [R] first segment slot of each range
    const int64_t *count;      // [R] elements of each range
    double *seg;               // segment results, [segments][rows]
    unsigned *counter;         // [R][rows], zero between launches
    float *out_prev, *out_last;
    int rows;                  // workers (worker scales) or 1 (server scales)
    int R;
    int out_stride_r, out_stride_row;  // out[r * stride_r + row * stride_row]
};

// Grid (R, rows, segments): worker scales use ranges = tensors and one row
// per worker; server scales use ranges = (tensor, chunk) and one row.
__global__ void __launch_bounds__(kScaleThreads) ob_scale_kernel(const __grid_constant__ ScaleParams P) {
    const int r = blockIdx.x, row = blockIdx.y, seg = blockIdx.z;
    const int lo = P.range_begin[r], hi = P.range_begin[r + 1];
    const int nseg = num_segments(hi - lo);
    if (seg >= nseg) return;
    double total = 0.0;
    const double *v = P.partial + (int64_t)row * P.n_tiles;
    double *seg_out = P.seg + ((int64_t)P.seg_base[r] * P.rows + (int64_t)row * nseg);
    if (!range_sum(v, lo, hi, seg, nseg, seg_out, P.counter + (int64_t)r * P.rows + row, &total))
        return;
    if (threadIdx.x == 0) {
        const float s = rms(total, P.count[r]);
        const int64_t o = (int64_t)r * P.out_stride_r + (int64_t)row * P.out_stride_row;
        P.out_prev[o] = s;
        P.out_last[o] = s;
    }
}

// ----------------------------------------------------------- server stage

constexpr int kTileWords = kTile / 32;  // sign words of one worker in a full tile

struct ServerParams {
    const Tile *tiles;
    const uint32_t *bits;   // [W][n_pad/32] this step's worker signs
    const float *s_w;       // [W][T] this step's worker scales
    float *y;               // [n_pad]: in y_prev (lazy e_s), out y
    const float *sp_prev;   // [T][W]: scale that decodes y_prev
    uint32_t *sbits;        // [n_pad/32]
    double *partial;        // [n_tiles]: sum of y^2 per tile
    int64_t n_pad;
    int W, T;
    float inv_w;            // 1/W when W is a power of two (then acc*inv_w == acc/W exactly)
    int w_pow2;
};

// Two independent IEEE round-to-nearest additions in one instruction
// (packed fp32 pair, sm_100a): (a0, a1) += (b0, b1), each lane exactly
// __fadd_rn.
__device__ __forceinline__ void add2_rn(float &a0, float &a1, float b0, float b1) {
    asm("{\n\t.reg .b64 ra, rb;\n\tmov.b64 ra, {%0, %1};\n\tmov.b64 rb, {%2, %3};\n\t"
        "add.rn.f32x2 ra, ra, rb;\n\tmov.b64 {%0, %1}, ra;\n\t}"
        : "+f"(a0), "+f"(a1)
        : "f"(b0), "f"(b1));
}

// [1BA, Proposed method, 3-4]: server j = tile.chunk receives every
// worker's words for its chunk (addressed in place: the exchange is an
// index into [W][words]) and forms
//   y = (sum over w in order of sign_w s_w) / W + e_s,
// with e_s decoded from (y_prev, s'_prev); then the sign bits of y and the
// tile's partial sum of y^2.  The tile's W word rows are staged in shared
// memory with one 16-byte load per thread, so the W-long sequential sum
// never waits on global memory.  FULL tiles (all 4096 elements real, the
// rule) skip every per-element bound check.
template <bool FULL>
__device__ __forceinline__ void server_tile(const ServerParams &P, const Tile &tile, int tile_id,
                                            const uint4 *staged, const uint32_t *scale_bits,
                                            double *red) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t word0 = tile.begin >> 5;

    float4 yo[kUnroll];
    int real[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int off = span_off(warp, lane, u);
        real[u] = FULL ? 4 : slot_real(tile.count, off);
        yo[u] = (FULL || real[u] > 0) ? ld_stream(P.y + tile.begin + off) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();

    const uint32_t *words = reinterpret_cast<const uint32_t *>(staged);
    const int shift = 4 * (lane & 7);  // bit of this lane's first element in its word
    float acc[kUnroll][4];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[u][k] = 0.0f;
#pragma unroll 4
    for (int w = 0; w < P.W; ++w) {
        const uint32_t sb = scale_bits[w];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            // this lane's 4 bits, inverted, at bits 0..3: element k's sign
            // bit is then (inv << (31 - k)) & 0x80000000 (a constant shift)
            const uint32_t inv = ~(words[w * kTileWords + (span_off(warp, lane, u) >> 5)] >> shift);
            const float v0 = __uint_as_float(((inv << 31) & 0x80000000u) | sb);
            const float v1 = __uint_as_float(((inv << 30) & 0x80000000u) | sb);
            const float v2 = __uint_as_float(((inv << 29) & 0x80000000u) | sb);
            const float v3 = __uint_as_float(((inv << 28) & 0x80000000u) | sb);
            add2_rn(acc[u][0], acc[u][1], v0, v1);
            add2_rn(acc[u][2], acc[u][3], v2, v3);
        }
    }

    const float wf = (float)P.W;
    const float sp = P.sp_prev[tile.tensor * P.W + tile.chunk];
    double ss[kUnroll];
    uint32_t out_words[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int off = span_off(warp, lane, u);
        uint32_t nibble = 0;
        ss[u] = 0.0;
        if (FULL || real[u] > 0) {
            float4 yn = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (FULL || k < real[u]) {
                    const float avg = P.w_pow2 ? __fmul_rn(acc[u][k], P.inv_w) : __fdiv_rn(acc[u][k], wf);
                    const float y = __fadd_rn(avg, decode_error(get(yo[u], k), sp));
                    ss[u] = __fma_rn((double)y, (double)y, ss[u]);
                    nibble |= (uint32_t)code_of(y) << k;
                    set(yn, k, y);
                }
            }
            st_stream(P.y + tile.begin + off, yn);
        }
        out_words[u] = gather_word(nibble, lane);
    }
    const uint32_t mine = collect_words(out_words, lane);
    if (lane < 4 * kUnroll && (FULL || (kUnroll * 128) * warp + 32 * lane < tile.count))
        P.sbits[word0 + 4 * kUnroll * warp + lane] = mine;
    double t = 0.0;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) t += ss[u];
    t = warp_sum(t);
    if (lane == 0) red[warp] = t;
    __syncthreads();
    if (tid == 0) {
        double a = 0.0;
#pragma unroll
        for (int k = 0; k < kWarps; ++k) a += red[k];
        P.partial[tile_id] = a;
    }
}

__global__ void __launch_bounds__(kThreads) ob_server_kernel(const __grid_constant__ ServerParams P) {
    extern __shared__ uint4 staged[];  // [W][kTileWords / 4]
    __shared__ double red[kWarps];
    __shared__ uint32_t scale_bits[OB_MAX_WORKERS];
    const int tile_id = blockIdx.x;
    const Tile tile = P.tiles[tile_id];
    const int tid = threadIdx.x;
    const int64_t words_per_worker = P.n_pad >> 5;
    const int64_t word0 = tile.begin >> 5;
    const int groups = (((tile.count + 31) >> 5) + 3) >> 2;  // 16-byte word groups with real elements

    for (int idx = tid; idx < P.W * (kTileWords / 4); idx += kThreads) {
        const int w = idx / (kTileWords / 4), q = idx % (kTileWords / 4);
        if (q < groups)
            staged[idx] = __ldcs(reinterpret_cast<const uint4 *>(P.bits + w * words_per_worker + word0) + q);
    }
    if (tid < P.W) scale_bits[tid] = __float_as_uint(P.s_w[tid * P.T + tile.tensor]);
    if (tile.count == kTile)
        server_tile<true>(P, tile, tile_id, staged, scale_bits, red);
    else
        server_tile<false>(P, tile, tile_id, staged, scale_bits, red);
}

// ------------------------------------------------------ gather and update

struct ApplyParams {
    const Tile *tiles;
    const uint32_t *sbits;  // [n_pad/32]
    const float *sp;        // [T][W] this step's server scales
    const float *d;         // [n_pad] frozen denominator
    float *p;               // [n_pad]
    float *m;               // [n_pad] dense momentum, or NULL to keep it as (sbits, sp)
    int W;
    float lr;
};

// [1BA, Proposed method, 1-2]: every worker decodes the gathered server
// words, m_hat = sign' s'_j, and takes a momentum SGD step preconditioned by
// the frozen denominator: p -= lr (m_hat / d); m = m_hat (m is left as the
// words and scales themselves unless a dense copy is asked for).
template <bool FULL>
__device__ __forceinline__ void apply_tile(const ApplyParams &P, const Tile &tile) {
    const int tid = threadIdx.x, lane = tid & 31;
    const uint32_t sb = __float_as_uint(P.sp[tile.tensor * P.W + tile.chunk]);
    const int shift = 4 * (lane & 7);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int off = 4 * (tid + kThreads * u);
        const int real = FULL ? 4 : slot_real(tile.count, off);
        if (!FULL && real == 0) continue;
        const int64_t i = tile.begin + off;
        const uint32_t inv = ~(__ldg(P.sbits + (i >> 5)) >> shift);
        const float4 d = ld_stream(P.d + i);
        float4 p = ld_stream(P.p + i);
        float4 m = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (FULL || k < real) {
                const float m_hat = __uint_as_float(((inv << (31 - k)) & 0x80000000u) | sb);
                const float delta = __fmul_rn(P.lr, __fdiv_rn(m_hat, get(d, k)));
                set(p, k, __fsub_rn(get(p, k), delta));
                set(m, k, m_hat);
            }
        }
        st_stream(P.p + i, p);
        if (P.m) st_stream(P.m + i, m);
    }
}

__global__ void __launch_bounds__(kThreads) ob_apply_kernel(const __grid_constant__ ApplyParams P) {
    const Tile tile = P.tiles[blockIdx.x];
    if (tile.count == kTile)
        apply_tile<true>(P, tile);
    else
        apply_tile<false>(P, tile);
}

// ------------------------------------------------- state decode for reads

// m = sign' s'_j from the server words, into out[i - out_base], over a run
// of tiles (padding left untouched).
__global__ void __launch_bounds__(kThreads) ob_decode_momentum_kernel(
    const Tile *tiles, int tile_base, const uint32_t *sbits, const float *sp, int W, float *out,
    int64_t out_base) {
    const Tile tile = tiles[tile_base + (int)blockIdx.x];
    const uint32_t sb = __float_as_uint(sp[tile.tensor * W + tile.chunk]);
    const int shift = 4 * (threadIdx.x & 7);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int off = 4 * ((int)threadIdx.x + kThreads * u);
        const int real = slot_real(tile.count, off);
        if (real == 0) continue;
        const uint32_t word = sbits[(tile.begin + off) >> 5];
        float4 m = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (k < real) set(m, k, signed_from_bit(word, shift + k, sb));
        *reinterpret_cast<float4 *>(out + (tile.begin + off - out_base)) = m;
    }
}

struct DecodeParams {
    const Tile *tiles;
    int tile_base;
    const float *x;        // [n_pad] lazy error values (x or y)
    const float *scales;   // scale of tile (t, j) at scales[t * stride_t + j * stride_j]
    int stride_t, stride_j;
    float *out;            // out[i - out_base] = decoded error
    int64_t out_base;
};

// e = fl(x - sign(x) s) over a run of tiles (padding left untouched).
__global__ void __launch_bounds__(kThreads) ob_decode_error_kernel(const __grid_constant__ DecodeParams P) {
    const Tile tile = P.tiles[P.tile_base + (int)blockIdx.x];
    const float s = P.scales[tile.tensor * P.stride_t + tile.chunk * P.stride_j];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int off = 4 * ((int)threadIdx.x + kThreads * u);
        const int real = slot_real(tile.count, off);
        if (real == 0) continue;
        const float4 x = ld_stream(P.x + tile.begin + off);
        float4 e = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (k < real) set(e, k, decode_error(get(x, k), s));
        *reinterpret_cast<float4 *>(P.out + (tile.begin + off - P.out_base)) = e;
    }
}

// ------------------------------- one-tensor compressor without allocation
//
// The worker stage's 1-bit compressor applied to a given x of n elements
// (no padding, any length): per-tile sums of squares and sign words, then
// s = ||x||_2 / sqrt(n), then e = x - sign(x) s.  Used by the entry point
// that takes its scratch from a static device array.  The tail of x is
// read element by element, so x needs no padding.

__device__ __forceinline__ float4 load_tail(const float *p, int real) {
    if (real == 4) return *reinterpret_cast<const float4 *>(p);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k = 0; k < real; ++k) set(v, k, p[k]);
    return v;
}

__device__ __forceinline__ void store_tail(float *p, const float4 &v, int real) {
    if (real == 4) {
        *reinterpret_cast<float4 *>(p) = v;
        return;
    }
    for (int k = 0; k < real; ++k) p[k] = get(v, k);
}

__global__ void __launch_bounds__(kThreads) ob_compress_partial_kernel(const float *x, int64_t n,
                                                                       uint32_t *bits,
                                                                       double *partial) {
    const int64_t begin = (int64_t)blockIdx.x * kTile;
    const int count = (int)(n - begin < kTile ? n - begin : (int64_t)kTile);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ double red[kWarps];
    double ss = 0.0;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int off = 4 * (tid + kThreads * u);
        const int real = slot_real(count, off);
        uint32_t nibble = 0;
        if (real > 0) {
            const float4 v = load_tail(x + begin + off, real);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (k < real) {
                    const float xk = get(v, k);
                    ss = __fma_rn((double)xk, (double)xk, ss);
                    nibble |= (uint32_t)code_of(xk) << k;
                }
            }
        }
        const uint32_t word = gather_word(nibble, lane);
        if ((lane & 7) == 0 && off < count) bits[(begin + off) >> 5] = word;
    }
    ss = warp_sum(ss);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    if (tid == 0) {
        double a = 0.0;
#pragma unroll
        for (int k = 0; k < kWarps; ++k) a += red[k];
        partial[blockIdx.x] = a;
    }
}

__global__ void __launch_bounds__(kScaleThreads) ob_compress_scale_kernel(const double *partial,
                                                                          int tiles, int64_t n,
                                                                          float *scale) {
    __shared__ double smem[kScaleThreads / 32];
    double acc = 0.0;
    for (int k = (int)threadIdx.x; k < tiles; k += kScaleThreads) acc += partial[k];
    acc = block_sum(acc, smem);
    if (threadIdx.x == 0)
        *scale = n > 0 ? __double2float_rn(__dsqrt_rn(__ddiv_rn(acc, (double)n))) : 0.0f;
}

__global__ void __launch_bounds__(kThreads) ob_compress_error_kernel(const float *x, int64_t n,
                                                                     const float *scale,
                                                                     float *err) {
    const int64_t begin = (int64_t)blockIdx.x * kTile;
    const int count = (int)(n - begin < kTile ? n - begin : (int64_t)kTile);
    const float s = *scale;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int off = 4 * ((int)threadIdx.x + kThreads * u);
        const int real = slot_real(count, off);
        if (real == 0) continue;
        const float4 v = load_tail(x + begin + off, real);
        float4 e;
#pragma unroll
        for (int k = 0; k < 4; ++k) set(e, k, decode_error(get(v, k), s));
        store_tail(err + begin + off, e, real);
    }
}

}  // namespace onebit
