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

}  // namespace onebit
