// kernels/apply.cuh -- Gather, decode and the preconditioned update.
//
// Part of libonebit (sm_100a); see onebit_kernels.cuh for the overview.
#pragma once

#include "common.cuh"

namespace onebit {

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
    // Split step with peer memory (n_shards > 0): the words of the tiles of
    // shard q (shard_end as in PackParams) are read from src_sbits[q], the
    // server words of the process serving it, and copied into sbits_copy
    // (this process's server words, which then hold every chunk's).
    int n_shards;
    int shard_end[OB_MAX_WORKERS];
    const uint32_t *src_sbits[OB_MAX_WORKERS];
    uint32_t *sbits_copy;
};

// [1BA, Proposed method, 1-2]: every worker decodes the gathered server
// words, m_hat = sign' s'_j, and takes a momentum SGD step preconditioned by
// the frozen denominator: p -= lr (m_hat / d); m = m_hat (m is left as the
// words and scales themselves unless a dense copy is asked for).
//
// The per-element IEEE division keeps the compiler from issuing a slot's
// loads ahead of the previous slot's arithmetic, and holding all slots in
// registers costs residency; so each thread first copies all its d and p
// slots into shared memory (cp.async, 32 KiB per CTA), then computes.
// lr: the step's learning rate (P.lr, or 1-bit LAMB's layerwise rate).
// With NORM the thread's sum of the new p^2 is returned (else 0).
// sbits: where the tile's server words are read (P.sbits, or the serving
// process's with peer memory); copy: where lane 8k of each group stores
// the word it read (NULL: nowhere).
template <bool FULL, bool NORM>
__device__ __forceinline__ double apply_tile(const ApplyParams &P, const Tile &tile, float4 (*sd)[kThreads],
                                             float4 (*spp)[kThreads], float lr, const uint32_t *sbits,
                                             uint32_t *copy) {
    const int tid = threadIdx.x, lane = tid & 31;
    const uint32_t sb = __float_as_uint(P.sp[tile.tensor * P.W + tile.chunk]);
    const int shift = 4 * (lane & 7);
    const uint64_t pol = evict_first_policy();
    uint32_t inv[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int off = 4 * (tid + kThreads * u);
        inv[u] = 0;
        if (FULL || off < tile.count) {
            const int64_t i = tile.begin + off;
            cp_async16(&sd[u][tid], P.d + i, pol);
            cp_async16(&spp[u][tid], P.p + i, pol);
            const uint32_t word = __ldg(sbits + (i >> 5));
            if (copy && (lane & 7) == 0) copy[i >> 5] = word;
            inv[u] = ~(word >> shift);
        }
    }
    cp_async_commit();
    cp_async_wait<0>();
    double pp = 0.0;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int off = 4 * (tid + kThreads * u);
        const int real = FULL ? 4 : slot_real(tile.count, off);
        if (!FULL && real == 0) continue;
        const int64_t i = tile.begin + off;
        const float4 d = sd[u][tid];
        float4 p = spp[u][tid];
        float4 m = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (FULL || k < real) {
                const float m_hat = __uint_as_float(((inv[u] << (31 - k)) & 0x80000000u) | sb);
                const float delta = __fmul_rn(lr, __fdiv_rn(m_hat, get(d, k)));
                const float pk = __fsub_rn(get(p, k), delta);
                set(p, k, pk);
                set(m, k, m_hat);
                if (NORM) pp = __fma_rn((double)pk, (double)pk, pp);
            }
        }
        st_stream(P.p + i, p);
        if (P.m) st_stream(P.m + i, m);
    }
    return pp;
}

__global__ void __launch_bounds__(kThreads) ob_apply_kernel(const __grid_constant__ ApplyParams P) {
    __shared__ float4 sd[kUnroll][kThreads];   // this thread's d slots
    __shared__ float4 spp[kUnroll][kThreads];  // and p slots
    const Tile tile = P.tiles[blockIdx.x];  // the work list is written once, at create
    grid_dependency_wait();
    allow_dependent_launch();
    const bool peer = P.n_shards > 0;
    const uint32_t *sbits = peer ? P.src_sbits[shard_of(blockIdx.x, P.n_shards, P.shard_end)] : P.sbits;
    uint32_t *copy = peer ? P.sbits_copy : nullptr;
    if (tile.count == kTile)
        apply_tile<true, false>(P, tile, sd, spp, P.lr, sbits, copy);
    else
        apply_tile<false, false>(P, tile, sd, spp, P.lr, sbits, copy);
}

}  // namespace onebit
