// kernels/scale.cuh -- Worker and server scales, finished inside the kernels that produce their partial sums.
//
// Part of libonebit (sm_100a); see onebit_kernels.cuh for the overview.
#pragma once

#include "common.cuh"

namespace onebit {

// ------------------------------------------------------------- scales
//
// A scale is sqrt(S / count) ([1BA, Proposed method, 3]: the 1-bit code's
// magnitude, the RMS of what it compresses), with S the sum of squares of
// one range of tiles: a tensor for the worker scales (one row per worker),
// a server chunk for the server scales (one row).  Every tile CTA writes
// its per-row partial sums, then takes part in a two-level reduction that
// needs no kernel of its own and never waits:
//   * a range is cut into segments of kScaleSegTiles tiles; the CTA that
//     arrives last at a segment (thread fence, then an atomic counter) sums
//     the segment's partials for every row;
//   * a range of one segment has its scales then; otherwise the CTA that
//     finishes the range's last segment sums the segment results and
//     writes the scales.
// Every addition's order is fixed by the layout alone (sum_rows), so the
// scales repeat run to run whatever the CTAs' timing.  The last arriver
// resets each counter to 0 for the next launch.  Ranges with no tiles (an
// empty tensor or server chunk) keep the scale they were given, 0.

constexpr int kScaleSegTiles = 512;

// Row sums of rows x [lo, hi) doubles, row r at base + r * row_stride,
// into out[r].  Warp g sums rows g, g + kWarps, ...: lane l adds entries
// lo + l, lo + l + 32, ... into four accumulators in turn, the accumulators
// are added pairwise and the lanes by a butterfly.  Ends with a barrier.
__device__ __forceinline__ void sum_rows(const double *base, int64_t row_stride, int rows, int lo,
                                         int hi, double *out) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int r = warp; r < rows; r += kWarps) {
        const double *v = base + (int64_t)r * row_stride;
        double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
        int k = lo + lane;
        for (; k + 96 < hi; k += 128) {
            a0 += __ldcg(v + k);
            a1 += __ldcg(v + k + 32);
            a2 += __ldcg(v + k + 64);
            a3 += __ldcg(v + k + 96);
        }
        for (; k < hi; k += 32) a0 += __ldcg(v + k);
        const double s = warp_sum((a0 + a1) + (a2 + a3));
        if (lane == 0) out[r] = s;
    }
    __syncthreads();
}

__device__ __forceinline__ float rms(double sum_sq, int64_t count) {
    return count > 0 ? __double2float_rn(__dsqrt_rn(__ddiv_rn(sum_sq, (double)count))) : 0.0f;
}

// The ranges a producing kernel reduces over, and where the segment sums
// and counters live.
struct RangeSums {
    const int *range_begin;    // [R+1] first tile of each range (absolute tile indices)
    const int *seg_base;       // [R] first segment slot of each range
    unsigned *seg_counter;     // [segment slots] arrivals, 0 between launches
    unsigned *range_counter;   // [R] finished segments, 0 between launches
    double *seg;               // segment sums: row r, slot q at seg[r * seg_stride + q]
    int seg_stride;
};

// Where a producing kernel finishes its scales: the reduction, then
// scale (range, row) = sqrt(sum / count[range]) at
// out[range * stride_r + row * stride_row].
struct ScaleEpilogue {
    RangeSums sums;
    const int64_t *count;      // [R] elements of each range
    float *out_prev, *out_last;
    int out_stride_r, out_stride_row;
};

// Called by every thread of a tile CTA once threads [0, rows) have stored
// the tile's partial sums partial[row * n_tiles + tile_id].  `range` is the
// tile's range; rows <= OB_MAX_WORKERS; kThreads threads.  The CTA that
// completes the range calls done(range, sums) in every thread, sums[r]
// being row r's total (shared memory); every other CTA returns without
// calling it.  The ranges' rows are summed in an order fixed by the layout.
template <class Done>
__device__ __forceinline__ void reduce_ranges(const RangeSums &E, const double *partial,
                                              int64_t n_tiles, int rows, int range, int tile_id,
                                              Done done) {
    __shared__ double sums[OB_MAX_WORKERS];
    __shared__ int last;
    const int tid = threadIdx.x;
    const int lo = E.range_begin[range], hi = E.range_begin[range + 1];
    const int nseg = (hi - lo + kScaleSegTiles - 1) / kScaleSegTiles;
    const int s = (tile_id - lo) / kScaleSegTiles;
    const int a = lo + s * kScaleSegTiles, b = min(hi, a + kScaleSegTiles);
    const int slot = E.seg_base[range] + s;
    __threadfence();  // this thread's partial sums before the arrival below
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        last = atomicAdd(&E.seg_counter[slot], 1u) == (unsigned)(b - a - 1);
    }
    __syncthreads();
    if (!last) return;
    __threadfence();  // the other CTAs' partial sums are visible from here
    sum_rows(partial, n_tiles, rows, a, b, sums);
    if (nseg > 1) {
        if (tid < rows) E.seg[(int64_t)tid * E.seg_stride + slot] = sums[tid];
        __threadfence();
        __syncthreads();
        if (tid == 0) {
            E.seg_counter[slot] = 0u;
            last = atomicAdd(&E.range_counter[range], 1u) == (unsigned)(nseg - 1);
        }
        __syncthreads();
        if (!last) return;
        __threadfence();
        sum_rows(E.seg + E.seg_base[range], E.seg_stride, rows, 0, nseg, sums);
        if (tid == 0) E.range_counter[range] = 0u;
    } else if (tid == 0) {
        E.seg_counter[slot] = 0u;
    }
    done(range, (const double *)sums);
}

__device__ __forceinline__ void finish_scales(const ScaleEpilogue &E, const double *partial,
                                              int64_t n_tiles, int rows, int range, int tile_id) {
    reduce_ranges(E.sums, partial, n_tiles, rows, range, tile_id,
                  [&](int r, const double *sums) {
                      const int tid = threadIdx.x;
                      if (tid < rows) {
                          const float sc = rms(sums[tid], E.count[r]);
                          const int64_t o = (int64_t)r * E.out_stride_r + (int64_t)tid * E.out_stride_row;
                          E.out_prev[o] = sc;
                          E.out_last[o] = sc;
                      }
                  });
}

}  // namespace onebit
