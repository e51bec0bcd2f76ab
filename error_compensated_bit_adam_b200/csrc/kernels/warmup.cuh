// kernels/warmup.cuh -- Warmup Adam step and the variance freeze.
//
// Part of libonebit (sm_100a); see onebit_kernels.cuh for the overview.
#pragma once

#include "common.cuh"

namespace onebit {

// ------------------------------------------------------------ warmup Adam

struct WarmupParams {
    const Tile *tiles;
    const float *g[OB_MAX_WORKERS];  // worker gradients, padded layout
    float *m, *v, *p;
    int W;
    float beta1, beta2, c1, c2, bc1, bc2, eps, lr;
};

// The direction of Adam's step from its moments: (m/bc1) / (sqrt(v/bc2) + eps).
__device__ __forceinline__ float adam_direction(const WarmupParams &P, float m, float v) {
    const float mhat = __fdiv_rn(m, P.bc1);
    const float vhat = __fdiv_rn(v, P.bc2);
    const float denom = __fadd_rn(__fsqrt_rn(vhat), P.eps);
    return __fdiv_rn(mhat, denom);
}

// Adam's moments of one element of the averaged gradient, updated in place
// (m = beta1 m + (1-beta1) gbar, v = beta2 v + (1-beta2) gbar^2), and the
// direction of its step.
__device__ __forceinline__ float adam_moments(const WarmupParams &P, float gbar, float &m, float &v) {
    m = __fadd_rn(__fmul_rn(P.beta1, m), __fmul_rn(P.c1, gbar));
    v = __fadd_rn(__fmul_rn(P.beta2, v), __fmul_rn(P.c2, __fmul_rn(gbar, gbar)));
    return adam_direction(P, m, v);
}

// The average of the W gradients of one float4 slot (a sequential fp32 sum
// in worker order from +0, then one IEEE division by W per element).
__device__ __forceinline__ float4 average_gradient(const WarmupParams &P, int64_t i) {
    const float wf = (float)P.W;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int w = 0; w < P.W; ++w) {
        const float4 g = ld_stream(P.g[w] + i);
        acc.x = __fadd_rn(acc.x, g.x);
        acc.y = __fadd_rn(acc.y, g.y);
        acc.z = __fadd_rn(acc.z, g.z);
        acc.w = __fadd_rn(acc.w, g.w);
    }
    return make_float4(__fdiv_rn(acc.x, wf), __fdiv_rn(acc.y, wf), __fdiv_rn(acc.z, wf),
                       __fdiv_rn(acc.w, wf));
}

// [1BA, Proposed method, 1]: one full-precision Adam step on the averaged
// gradient, elementwise.
__global__ void __launch_bounds__(kThreads) ob_warmup_kernel(const __grid_constant__ WarmupParams P) {
    const Tile tile = P.tiles[blockIdx.x];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int off = 4 * ((int)threadIdx.x + kThreads * u);
        const int real = slot_real(tile.count, off);
        if (real == 0) continue;
        const int64_t i = tile.begin + off;
        const float4 gbar = average_gradient(P, i);
        float4 m = ld_stream(P.m + i), v = ld_stream(P.v + i), p = ld_stream(P.p + i);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (k >= real) break;  // padding keeps its values
            float mk = get(m, k), vk = get(v, k);
            const float r = adam_moments(P, get(gbar, k), mk, vk);
            const float delta = __fmul_rn(P.lr, r);
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
    // every slot's load first, so that the four are in flight together
    // while the divides and square roots run
    float4 x[kUnroll];
    int real[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int off = 4 * ((int)threadIdx.x + kThreads * u);
        real[u] = slot_real(tile.count, off);
        x[u] = real[u] > 0 ? ld_stream(v + tile.begin + off) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        if (real[u] == 0) continue;
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (k < real[u]) set(x[u], k, __fadd_rn(__fsqrt_rn(__fdiv_rn(get(x[u], k), bc2)), eps));
        st_stream(v + tile.begin + 4 * ((int)threadIdx.x + kThreads * u), x[u]);
    }
}

}  // namespace onebit
