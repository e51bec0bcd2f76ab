// kernels/state.cuh -- Decoders used when the host reads lazily stored state.
//
// Part of libonebit (sm_100a); see onebit_kernels.cuh for the overview.
#pragma once

#include "common.cuh"

namespace onebit {

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

}  // namespace onebit
