// kernels/scale.cuh -- Range sums of per-tile partial sums: the worker and server scales, and 1-bit LAMB's norms.
//
// Part of libonebit (sm_100a); see onebit_kernels.cuh for the overview.
#pragma once

#include "common.cuh"

namespace onebit {

// ------------------------------------------------------------- scales
//
// A scale is sqrt(S / count) ([1BA, Proposed method, 3]: the 1-bit code's
// magnitude, the RMS of what it compresses), with S the sum of the per-tile
// partial sums of one range of tiles (a tensor for the worker scales, a
// server chunk for the server scales).  A range is cut into segments of
// kScaleSegTiles tiles; one CTA sums one segment, and the CTA that finishes
// last for the range sums the segment results in segment order.  The order
// of every addition is fixed by the layout, so the scales repeat run to
// run.  The last CTA is found with a per-range counter (thread fence, then
// atomic increment; it resets the counter), so nothing ever waits.
//
// The same kernel also returns plain range sums (out_sum), for 1-bit
// LAMB's norms.
//
// The reduction is a kernel of its own on purpose: finishing it in the
// tail of the tile kernels that produce the partial sums (fence, atomic
// arrival, barrier at the end of every CTA) held each CTA and its shared
// memory past its last store and cost 15% of the worker stage and 20% of
// the server stage on the B200, against about 20 us for these launches.

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
    float *out_prev, *out_last;  // scales, when out_sum is NULL
    double *out_sum;           // plain range sums instead, when not NULL
    int rows;                  // workers (worker scales) or 1 (server scales)
    int R;
    int out_stride_r, out_stride_row;  // out[r * stride_r + row * stride_row]
};

// Grid (R, rows, segments): worker scales use ranges = tensors and one row
// per worker; server scales use ranges = (tensor, chunk) and one row.
__global__ void __launch_bounds__(kScaleThreads) ob_scale_kernel(const __grid_constant__ ScaleParams P) {
    const int r = blockIdx.x, row = blockIdx.y, seg = blockIdx.z;
    grid_dependency_wait();
    allow_dependent_launch();
    const int lo = P.range_begin[r], hi = P.range_begin[r + 1];
    const int nseg = num_segments(hi - lo);
    if (seg >= nseg) return;
    double total = 0.0;
    const double *v = P.partial + (int64_t)row * P.n_tiles;
    double *seg_out = P.seg + ((int64_t)P.seg_base[r] * P.rows + (int64_t)row * nseg);
    if (!range_sum(v, lo, hi, seg, nseg, seg_out, P.counter + (int64_t)r * P.rows + row, &total))
        return;
    if (threadIdx.x == 0) {
        const int64_t o = (int64_t)r * P.out_stride_r + (int64_t)row * P.out_stride_row;
        if (P.out_sum) {
            P.out_sum[o] = total;
        } else {
            const float s = rms(total, P.count[r]);
            P.out_prev[o] = s;
            P.out_last[o] = s;
        }
    }
}

}  // namespace onebit
