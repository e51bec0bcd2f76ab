// kernels/pack.cuh -- Worker stage: momentum, error feedback, 1-bit compression of every worker.
//
// Part of libonebit (sm_100a); see onebit_kernels.cuh for the overview.
#pragma once

#include "common.cuh"

namespace onebit {

// ----------------------------------------------------------- worker stage

struct PackParams {
    const Tile *tiles;
    int tile_base;                   // tile of blockIdx.x == 0
    int n_tiles;                     // total tiles (row length of partial)
    const float *m;                  // [n_pad] dense momentum (when m_dense)
    const uint32_t *m_bits;          // [n_pad/32] last step's server signs (when !m_dense)
    const float *m_scale;            // [T][chunks] last step's server scales (when !m_dense)
    int m_dense;
    int chunks;                      // server chunks per tensor (the context's W, whatever W below is)
    const float *g[OB_MAX_WORKERS];  // element i of worker w at g[w][i - g_offset]
    int64_t g_offset;
    float *x;                        // [W][n_pad]: in x_prev (lazy e_w), out x
    uint32_t *bits;                  // [W][n_pad/32]
    const float *s_prev;             // [W][T]: scale that decodes x_prev
    double *partial;                 // [W][n_tiles]: sum of x^2 per tile
    int64_t n_pad;
    int W, T;
    float beta1, c1;
    // Split step with peer memory (n_shards > 0): the words of the tiles
    // below shard_end[q] (absolute tile ids, ascending) and not below
    // shard_end[q-1] go to dest[q] -- the worker rows of the process serving
    // shard q, offset to this launch's first worker -- instead of `bits`.
    int n_shards;
    int shard_end[OB_MAX_WORKERS];
    uint32_t *dest[OB_MAX_WORKERS];
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
    const Tile tile = P.tiles[tile_id];  // the work list is written once, at create
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ double red[kWarps][OB_MAX_WORKERS];
    grid_dependency_wait();
    allow_dependent_launch();

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
        const uint32_t sb = __float_as_uint(P.m_scale[tile.tensor * P.chunks + tile.chunk]);
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
    uint32_t *const bits = P.n_shards > 0 ? P.dest[shard_of(tile_id, P.n_shards, P.shard_end)] : P.bits;
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
        uint32_t *bw = bits + (int64_t)w * words_per_worker + (tile.begin >> 5);
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

}  // namespace onebit
