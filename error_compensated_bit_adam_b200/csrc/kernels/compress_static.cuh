// kernels/compress_static.cuh -- The one-tensor compressor behind the allocation-free entry point.
//
// Part of libonebit (sm_100a); see onebit_kernels.cuh for the overview.
#pragma once

#include "scale.cuh"

namespace onebit {

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
