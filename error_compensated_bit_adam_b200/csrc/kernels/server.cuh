// kernels/server.cuh -- Server stage: average of the workers' compressed momenta, server error, re-compression.
//
// Part of libonebit (sm_100a); see onebit_kernels.cuh for the overview.
#pragma once

#include "common.cuh"

namespace onebit {

// ----------------------------------------------------------- server stage

constexpr int kTileWords = kTile / 32;  // sign words of one worker in a full tile

// The first kSumTableWorkers workers' part of the sequential sum comes from
// a table: with the scales s_0..s_7 of the tile's tensor fixed, the running
// sum after those workers depends only on their 8 sign bits, so the CTA
// tabulates all 256 values once and each element looks its value up.
constexpr int kSumTableWorkers = 8;
constexpr int kSumTableSize = 1 << kSumTableWorkers;

// Each lane owns 2 slots of 8 consecutive elements: slot j of lane l of
// warp v is elements [2048 j + 256 v + 8 l, +8), i.e. byte l % 4 of the
// tile's sign word 64 j + 8 v + l / 4 (of every worker), and its inputs and
// outputs are one 32-byte access each.
constexpr int kSlotElems = 8;
constexpr int kSlots = kTile / (kThreads * kSlotElems);
static_assert(kSlots == 2, "server slots");

__device__ __forceinline__ int server_off(int warp, int lane, int j) {
    return (kThreads * kSlotElems) * j + (32 * kSlotElems) * warp + kSlotElems * lane;
}

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

// 32-byte streaming accesses (sm_100): one slot of 8 floats.
__device__ __forceinline__ void ld_stream8(const float *p, float (&v)[8]) {
    asm("ld.global.cs.v8.f32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
        : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
        : "l"(p));
}
__device__ __forceinline__ void st_stream8(float *p, const float (&v)[8]) {
    asm volatile("st.global.cs.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "f"(v[0]), "f"(v[1]),
                 "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
}

// Transpose the 8x8 bit matrix held in (lo, hi), row i = byte i (bytes
// 0..3 in lo, 4..7 in hi), column k = bit k of every byte: afterwards
// byte k holds what was bit k of bytes 0..7 (as its bits 0..7).  Three
// delta swaps: bits within 2x2, 4x4 and 8x8 blocks.
__device__ __forceinline__ void transpose8x8(uint32_t &lo, uint32_t &hi) {
    uint32_t t;
    t = ((lo >> 7) ^ lo) & 0x00AA00AAu;
    lo = lo ^ t ^ (t << 7);
    t = ((hi >> 7) ^ hi) & 0x00AA00AAu;
    hi = hi ^ t ^ (t << 7);
    t = ((lo >> 14) ^ lo) & 0x0000CCCCu;
    lo = lo ^ t ^ (t << 14);
    t = ((hi >> 14) ^ hi) & 0x0000CCCCu;
    hi = hi ^ t ^ (t << 14);
    t = ((hi << 4) ^ lo) & 0xF0F0F0F0u;
    lo = lo ^ t;
    hi = hi ^ (t >> 4);
}

// [1BA, Proposed method, 3-4]: server j = tile.chunk receives every
// worker's words for its chunk (addressed in place: the exchange is an
// index into [W][words]) and forms
//   y = (sum over w in order of sign_w s_w) / W + e_s,
// with e_s decoded from (y_prev, s'_prev); then the sign bits of y and the
// tile's partial sum of y^2.  The sum is the sequential fp32 sum from +0
// in worker order: its first min(W, 8) terms from the table, the rest
// added one by one (two elements per packed add).  FULL tiles (all 4096
// elements real, the rule) skip every per-element bound check.
template <bool FULL, bool POW2>
__device__ __forceinline__ void server_tile(const ServerParams &P, const Tile &tile, int tile_id,
                                            const float (&yo)[kSlots][kSlotElems], float sp, const uint32_t *words,
                                            const float *table, const uint32_t *scale_bits, double *red) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t word0 = tile.begin >> 5;
    const int b = lane & 3;  // the lane's byte of each sign word

    int real[kSlots];
#pragma unroll
    for (int j = 0; j < kSlots; ++j)
        real[j] = FULL ? kSlotElems : min(kSlotElems, max(0, tile.count - server_off(warp, lane, j)));
    __syncthreads();  // the staged words and the table are in

    const int G = P.W < kSumTableWorkers ? P.W : kSumTableWorkers;
    // byte b of each of two words into bytes 0 and 1
    const uint32_t pick = (uint32_t)b | ((uint32_t)(4 + b) << 4);
    const float wf = (float)P.W;
    double ss = 0.0;
    uint32_t out_word[kSlots];
#pragma unroll
    for (int j = 0; j < kSlots; ++j) {
        const int off = server_off(warp, lane, j);
        const int q = off >> 5;  // the slot's sign word within the tile
        uint32_t wv[kSumTableWorkers];
#pragma unroll
        for (int w = 0; w < kSumTableWorkers; ++w) wv[w] = w < G ? words[w * kTileWords + q] : 0u;
        // byte w of (lo, hi): worker w's byte b; transposed, byte k: the 8
        // workers' sign bits of element k (bit w = worker w)
        uint32_t lo = __byte_perm(__byte_perm(wv[0], wv[1], pick), __byte_perm(wv[2], wv[3], pick), 0x5410);
        uint32_t hi = __byte_perm(__byte_perm(wv[4], wv[5], pick), __byte_perm(wv[6], wv[7], pick), 0x5410);
        transpose8x8(lo, hi);
        float acc[kSlotElems];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            acc[k] = table[(lo >> (8 * k)) & 0xFFu];
            acc[4 + k] = table[(hi >> (8 * k)) & 0xFFu];
        }
#pragma unroll 4
        for (int w = kSumTableWorkers; w < P.W; ++w) {
            const uint32_t sb = scale_bits[w];
            // the lane's 8 bits, inverted, at bits 0..7: element k's sign
            // bit is then (inv << (31 - k)) & 0x80000000 (a constant shift)
            const uint32_t inv = ~(words[w * kTileWords + q] >> (8 * b));
            float v[kSlotElems];
#pragma unroll
            for (int k = 0; k < kSlotElems; ++k) v[k] = __uint_as_float(((inv << (31 - k)) & 0x80000000u) | sb);
#pragma unroll
            for (int k = 0; k < kSlotElems; k += 2) add2_rn(acc[k], acc[k + 1], v[k], v[k + 1]);
        }
        uint32_t code = 0;
        if (FULL || real[j] > 0) {
            float yn[kSlotElems];
#pragma unroll
            for (int k = 0; k < kSlotElems; ++k) {
                yn[k] = 0.0f;
                if (FULL || k < real[j]) {
                    const float avg = POW2 ? __fmul_rn(acc[k], P.inv_w) : __fdiv_rn(acc[k], wf);
                    const float y = __fadd_rn(avg, decode_error(yo[j][k], sp));
                    ss = __fma_rn((double)y, (double)y, ss);
                    code |= (uint32_t)code_of(y) << k;
                    yn[k] = y;
                }
            }
            st_stream8(P.y + tile.begin + off, yn);
        }
        // the 4 lanes of a word hold its 4 bytes
        uint32_t word = code << (8 * b);
        word |= __shfl_xor_sync(kFull, word, 1);
        word |= __shfl_xor_sync(kFull, word, 2);
        out_word[j] = word;
    }
#pragma unroll
    for (int j = 0; j < kSlots; ++j) {
        const int q = server_off(warp, lane, j) >> 5;
        if (b == 0 && (FULL || 32 * q < tile.count)) P.sbits[word0 + q] = out_word[j];
    }
    const double t = warp_sum(ss);
    if (lane == 0) red[warp] = t;
    __syncthreads();
    if (tid == 0) {
        double a = 0.0;
#pragma unroll
        for (int k = 0; k < kWarps; ++k) a += red[k];
        P.partial[tile_id] = a;
    }
}

// Six CTAs per SM (at most 40 registers a thread): the per-tile prologue
// (the word rows, the scales, the table) waits on memory, and the more
// CTAs are resident, the more of that wait other CTAs' arithmetic covers.
constexpr int kServerCtasPerSm = 6;

__global__ void __launch_bounds__(kThreads, kServerCtasPerSm) ob_server_kernel(const __grid_constant__ ServerParams P) {
    extern __shared__ uint4 staged[];  // [W][kTileWords / 4]
    __shared__ float table[kSumTableSize];
    __shared__ double red[kWarps];
    __shared__ uint32_t scale_bits[OB_MAX_WORKERS];
    const int tile_id = P.tile_base + (int)blockIdx.x;
    const Tile tile = P.tiles[tile_id];  // the work list is written once, at create
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // y_prev and s'_prev are read before waiting for the previous kernel:
    // they were written by an earlier step's server stage (or the freeze,
    // or a state write), never by the kernel this launch waits on.  Every
    // kernel of the library that lets its successor start early
    // (allow_dependent_launch) first waits for its own predecessor, so when
    // this kernel starts, every kernel before its immediate predecessor has
    // completed.
    float yo[kSlots][kSlotElems];
#pragma unroll
    for (int j = 0; j < kSlots; ++j) {
        const int off = server_off(warp, lane, j);
        if (off < tile.count) {
            ld_stream8(P.y + tile.begin + off, yo[j]);
        } else {
#pragma unroll
            for (int k = 0; k < kSlotElems; ++k) yo[j][k] = 0.0f;
        }
    }
    const float sp = P.sp_prev[tile.tensor * P.W + tile.chunk];
    grid_dependency_wait();
    allow_dependent_launch();
    const int64_t words_per_worker = P.n_pad >> 5;
    const int64_t word0 = tile.begin >> 5;
    const int groups = (((tile.count + 31) >> 5) + 3) >> 2;  // 16-byte word groups with real elements

    // the word rows straight into shared memory (awaited before the barrier)
    const uint64_t pol = evict_first_policy();
    for (int idx = tid; idx < P.W * (kTileWords / 4); idx += kThreads) {
        const int w = idx / (kTileWords / 4), q = idx % (kTileWords / 4);
        if (q < groups)
            cp_async16(staged + idx, reinterpret_cast<const uint4 *>(P.bits + w * words_per_worker + word0) + q, pol);
    }
    cp_async_commit();
    if (tid < P.W) scale_bits[tid] = __float_as_uint(P.s_w[tid * P.T + tile.tensor]);
    // Table entry e: the sequential fp32 sum from +0, over the first
    // min(W, 8) workers in order, of +s_w where bit w of e is set, else -s_w
    // (bits of workers past W are ignored).
    {
        static_assert(kSumTableSize == kThreads, "one table entry per thread");
        const int G = P.W < kSumTableWorkers ? P.W : kSumTableWorkers;
        float s[kSumTableWorkers];
#pragma unroll
        for (int w = 0; w < kSumTableWorkers; ++w) s[w] = w < G ? P.s_w[w * P.T + tile.tensor] : 0.0f;
        float a = 0.0f;
#pragma unroll
        for (int w = 0; w < kSumTableWorkers; ++w)
            if (w < G) a = __fadd_rn(a, ((tid >> w) & 1) ? s[w] : -s[w]);
        table[tid] = a;
    }
    const uint32_t *words = reinterpret_cast<const uint32_t *>(staged);
    cp_async_wait<0>();
    if (tile.count == kTile) {
        if (P.w_pow2)
            server_tile<true, true>(P, tile, tile_id, yo, sp, words, table, scale_bits, red);
        else
            server_tile<true, false>(P, tile, tile_id, yo, sp, words, table, scale_bits, red);
    } else {
        if (P.w_pow2)
            server_tile<false, true>(P, tile, tile_id, yo, sp, words, table, scale_bits, red);
        else
            server_tile<false, false>(P, tile, tile_id, yo, sp, words, table, scale_bits, red);
    }
}

}  // namespace onebit
