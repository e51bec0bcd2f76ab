// kernels/server.cuh -- Server stage: average of the workers' compressed momenta, server error, re-compression.
//
// Part of libonebit (sm_100a); see onebit_kernels.cuh for the overview.
#pragma once

#include "common.cuh"

namespace onebit {

// ----------------------------------------------------------- server stage

constexpr int kTileWords = kTile / 32;  // sign words of one worker in a full tile

struct ServerParams {
    const Tile *tiles;
    int tile_base;          // tile of blockIdx.x == 0 (partial sums indexed by the absolute tile)
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
    const int tile_id = P.tile_base + (int)blockIdx.x;
    const Tile tile = P.tiles[tile_id];  // the work list is written once, at create
    const int tid = threadIdx.x;
    grid_dependency_wait();
    allow_dependent_launch();
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

}  // namespace onebit
