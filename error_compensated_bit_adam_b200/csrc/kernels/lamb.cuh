// kernels/lamb.cuh -- 1-bit LAMB: layerwise trust ratios for the warmup and the compressed update.
//
// Part of libonebit (sm_100a); see onebit_kernels.cuh for the overview.
//
// The 1-bit LAMB review page ("1-bit LAMB: Communication Efficient
// Large-Scale Large-Batch Training with LAMB's Convergence Speed",
// Abstract) keeps LAMB's adaptive layerwise learning rates while the
// momentum is exchanged compressed.  Reading taken (the page prints no
// rule): each tensor's step is scaled by LAMB's trust ratio
//   ratio = ||p|| / ||u||   (1 when either norm is 0),
// u being Adam's direction in the warmup and m_hat / d in the compression
// phase (m_hat the decoded averaged momentum every worker holds after the
// gather, d the frozen denominator); the ratio is recomputed every step.
// The other reading, the ratios of the last warmup step kept at the freeze
// like the variance, makes the compressed update read the stored ratio
// (LambApplyParams::fixed_ratio) and needs none of the norms below.
//
// In the compression phase ||u||^2 = sum_j s'_j^2 D_j over the tensor's
// server chunks j, with D_j = sum over the chunk of (1/d)^2: d is frozen,
// so D_j is computed once (ob_lamb_norms_kernel, at the freeze) and every
// step needs only the chunk scales.  ||p||^2 is summed by the update kernel
// as it writes p (for the next step), and by ob_lamb_norms_kernel whenever
// p was changed otherwise (warmup, freeze, a state write).  Every kernel
// here leaves per-tile partial sums; ob_scale_kernel (scale.cuh) adds them
// per tensor or chunk in its fixed order.
#pragma once

#include "common.cuh"
#include "scale.cuh"
#include "warmup.cuh"
#include "apply.cuh"

namespace onebit {

__device__ __forceinline__ float trust_ratio(double p_sq, double u_sq) {
    return (p_sq > 0.0 && u_sq > 0.0) ? __double2float_rn(__dsqrt_rn(__ddiv_rn(p_sq, u_sq))) : 1.0f;
}

// Fixed-order sum over the CTA's kThreads threads of two values (results
// valid in thread 0).
__device__ __forceinline__ void block_sum2(double &a, double &b, double (*red)[2]) {
    a = warp_sum(a);
    b = warp_sum(b);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) {
        red[warp][0] = a;
        red[warp][1] = b;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        a = 0.0;
        b = 0.0;
        for (int k = 0; k < kWarps; ++k) {
            a += red[k][0];
            b += red[k][1];
        }
    }
}

// ---------------------------------------------------------- LAMB warmup

struct LambWarmupParams {
    WarmupParams w;
    double *partial;      // [2][n_tiles]: per tile, sum of p^2 (before the step) and of r^2
    int64_t n_tiles;
    const double *sums;   // [2][T]: the tensors' ||p||^2 and ||r||^2 (for the step kernel)
    int T;
    const int *tensor_tile_begin;  // [T+1]
    float *ratio;         // [T] out: the tensors' trust ratios
};

// First half of a LAMB warmup step: Adam's moments (written back) and the
// tile's partial sums of p^2 (the parameters before the step) and of r^2
// (Adam's direction).
__global__ void __launch_bounds__(kThreads) ob_lamb_moments_kernel(const __grid_constant__ LambWarmupParams P) {
    const int tile_id = (int)blockIdx.x;
    const Tile tile = P.w.tiles[tile_id];
    __shared__ double red[kWarps][2];
    double pp = 0.0, rr = 0.0;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int off = 4 * ((int)threadIdx.x + kThreads * u);
        const int real = slot_real(tile.count, off);
        if (real == 0) continue;
        const int64_t i = tile.begin + off;
        const float4 gbar = average_gradient(P.w, i);
        float4 m = ld_stream(P.w.m + i), v = ld_stream(P.w.v + i);
        const float4 p = ld_stream(P.w.p + i);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (k >= real) break;
            float mk = get(m, k), vk = get(v, k);
            const float r = adam_moments(P.w, get(gbar, k), mk, vk);
            set(m, k, mk);
            set(v, k, vk);
            pp = __fma_rn((double)get(p, k), (double)get(p, k), pp);
            rr = __fma_rn((double)r, (double)r, rr);
        }
        st_stream(P.w.m + i, m);
        st_stream(P.w.v + i, v);
    }
    block_sum2(pp, rr, red);
    if (threadIdx.x == 0) {
        P.partial[tile_id] = pp;
        P.partial[P.n_tiles + tile_id] = rr;
    }
}

// Second half, once the sums are reduced per tensor: ratio_t =
// ||p|| / ||r||, then p -= (lr * ratio_t) * r, r recomputed from the stored
// moments with the same operations (so the same values).
__global__ void __launch_bounds__(kThreads) ob_lamb_step_kernel(const __grid_constant__ LambWarmupParams P) {
    const int tile_id = (int)blockIdx.x;
    const Tile tile = P.w.tiles[tile_id];
    const int t = tile.tensor;
    const float ratio = trust_ratio(P.sums[t], P.sums[P.T + t]);
    if (threadIdx.x == 0 && tile_id == P.tensor_tile_begin[t]) P.ratio[t] = ratio;
    const float lr_t = __fmul_rn(P.w.lr, ratio);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int off = 4 * ((int)threadIdx.x + kThreads * u);
        const int real = slot_real(tile.count, off);
        if (real == 0) continue;
        const int64_t i = tile.begin + off;
        const float4 m = ld_stream(P.w.m + i), v = ld_stream(P.w.v + i);
        float4 p = ld_stream(P.w.p + i);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (k >= real) break;
            const float r = adam_direction(P.w, get(m, k), get(v, k));
            set(p, k, __fsub_rn(get(p, k), __fmul_rn(lr_t, r)));
        }
        st_stream(P.w.p + i, p);
    }
}

// ------------------------------------------------------------- the norms

struct LambNormsParams {
    const Tile *tiles;
    const float *d, *p;
    double *partial_d;  // [n_tiles] per tile, sum of (1/d)^2 (when want_d)
    double *partial_p;  // [n_tiles] per tile, sum of p^2 (when want_p)
    int want_d, want_p;
};

// Per-tile sums for D_j = sum over chunk j of (1/d)^2 and for ||p||^2.
__global__ void __launch_bounds__(kThreads) ob_lamb_norms_kernel(const __grid_constant__ LambNormsParams P) {
    const int tile_id = (int)blockIdx.x;
    const Tile tile = P.tiles[tile_id];
    __shared__ double red[kWarps][2];
    grid_dependency_wait();
    double dd = 0.0, pp = 0.0;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int off = 4 * ((int)threadIdx.x + kThreads * u);
        const int real = slot_real(tile.count, off);
        if (real == 0) continue;
        const int64_t i = tile.begin + off;
        const float4 d = P.want_d ? ld_stream(P.d + i) : make_float4(1.f, 1.f, 1.f, 1.f);
        const float4 p = P.want_p ? ld_stream(P.p + i) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (k >= real) break;
            const double q = __ddiv_rn(1.0, (double)get(d, k));
            dd = __dadd_rn(dd, __dmul_rn(q, q));
            pp = __fma_rn((double)get(p, k), (double)get(p, k), pp);
        }
    }
    block_sum2(dd, pp, red);
    if (threadIdx.x == 0) {
        if (P.want_d) P.partial_d[tile_id] = dd;
        if (P.want_p) P.partial_p[tile_id] = pp;
    }
}

// ------------------------------------------------- the compressed update

struct LambApplyParams {
    ApplyParams a;
    const int *tensor_tile_begin;  // [T+1]
    const double *pnorm;  // [T]: ||p||^2 before this step
    const double *dnorm;  // [T][W]: D_j
    float *ratio;         // [T] out (in, when fixed_ratio)
    double *partial;      // [n_tiles]: per tile, sum of the new p^2 (the next step's ||p||^2)
    int fixed_ratio;      // the ratios kept at the freeze: read ratio, no norms, no partial
};

// [1BA, Proposed method, 1-2] with the 1-bit LAMB page's layerwise rates:
// the gather and update of ob_apply_kernel with lr_t = lr * ratio_t, where
// ratio_t = ||p|| / ||m_hat / d|| is formed by every CTA of tensor t from
// the tensor's W chunk scales (in chunk order) and ||p||^2; and the tile's
// partial sum of the new p^2.
__global__ void __launch_bounds__(kThreads) ob_lamb_apply_kernel(const __grid_constant__ LambApplyParams P) {
    __shared__ float4 sd[kUnroll][kThreads];
    __shared__ float4 spp[kUnroll][kThreads];
    __shared__ double red[kWarps][2];
    const int tile_id = (int)blockIdx.x;
    const Tile tile = P.a.tiles[tile_id];
    grid_dependency_wait();
    allow_dependent_launch();
    const int t = tile.tensor, W = P.a.W;
    const bool peer = P.a.n_shards > 0;
    const uint32_t *sbits = peer ? P.a.src_sbits[shard_of(tile_id, P.a.n_shards, P.a.shard_end)] : P.a.sbits;
    uint32_t *copy = peer ? P.a.sbits_copy : nullptr;
    if (P.fixed_ratio) {  // the ratio kept at the freeze
        const float lr_t = __fmul_rn(P.a.lr, P.ratio[t]);
        if (tile.count == kTile)
            apply_tile<true, false>(P.a, tile, sd, spp, lr_t, sbits, copy);
        else
            apply_tile<false, false>(P.a, tile, sd, spp, lr_t, sbits, copy);
        return;
    }
    double u_sq = 0.0;
    for (int j = 0; j < W; ++j) {
        const double s = (double)P.a.sp[t * W + j];
        u_sq = __dadd_rn(u_sq, __dmul_rn(__dmul_rn(s, s), P.dnorm[t * W + j]));
    }
    const float ratio = trust_ratio(P.pnorm[t], u_sq);
    if (threadIdx.x == 0 && tile_id == P.tensor_tile_begin[t]) P.ratio[t] = ratio;
    const float lr_t = __fmul_rn(P.a.lr, ratio);
    double pp;
    if (tile.count == kTile)
        pp = apply_tile<true, true>(P.a, tile, sd, spp, lr_t, sbits, copy);
    else
        pp = apply_tile<false, true>(P.a, tile, sd, spp, lr_t, sbits, copy);
    double unused = 0.0;
    block_sum2(pp, unused, red);
    if (threadIdx.x == 0) P.partial[tile_id] = pp;
}

}  // namespace onebit
