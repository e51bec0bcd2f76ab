// kernels/common.cuh -- Constants, the tile descriptor and device helpers shared by every kernel.
//
// Part of libonebit (sm_100a); see onebit_kernels.cuh for the overview.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../../include/onebit.h"

namespace onebit {


constexpr int kThreads = 256;              // threads per CTA of the tile kernels
constexpr int kWarps = kThreads / 32;
constexpr int kUnroll = 4;                 // float4 slots per thread per tile
constexpr int kTile = kThreads * 4 * kUnroll;  // 4096 elements per tile
constexpr int kScaleThreads = 256;         // threads of the scale kernels
constexpr int kPackStages = 2;             // workers in flight in the worker-stage pipeline
constexpr int kPackSmemBytes = kPackStages * 2 * kUnroll * kThreads * 16;  // 64 KiB: 3 CTAs per SM
constexpr unsigned kFull = 0xffffffffu;

// One unit of work: up to kTile consecutive elements of one tensor that all
// belong to one server chunk.  begin is the padded-layout element offset of
// the tile's first element (a multiple of 128); count is the number of real
// (non-padding) elements.
struct Tile {
    int64_t begin;
    int32_t count;
    int32_t tensor;
    int32_t chunk;
    int32_t reserved;
};
static_assert(sizeof(Tile) == 24, "Tile layout");
static_assert(kWarps * kUnroll * 128 == kTile, "warp spans cover a tile");
static_assert(kUnroll * 4 <= 32, "a warp's sign words fit one store");

// ---------------------------------------------------------------- helpers

__device__ __forceinline__ float signed_scale(bool plus, float s) { return plus ? s : -s; }

// The 1-bit code: +1 for x >= 0 (so +0.0 and -0.0 give +1), else -1.
__device__ __forceinline__ bool code_of(float x) { return x >= 0.0f; }

// Error feedback stored lazily as (x, s): e = fl(x - sign(x) s).
__device__ __forceinline__ float decode_error(float x, float s) {
    return __fsub_rn(x, signed_scale(code_of(x), s));
}

// +-s as a float, from a sign word: bit b of `word` set -> +s, clear -> -s.
// s >= 0, so only the sign bit changes: (~word << (31 - b)) keeps the
// inverted bit in bit 31.
__device__ __forceinline__ float signed_from_bit(uint32_t word, int b, uint32_t s_bits) {
    return __uint_as_float(((~word << (31 - b)) & 0x80000000u) | s_bits);
}

__device__ __forceinline__ float get(const float4 &v, int k) {
    return k == 0 ? v.x : (k == 1 ? v.y : (k == 2 ? v.z : v.w));
}
__device__ __forceinline__ void set(float4 &v, int k, float f) {
    if (k == 0) v.x = f; else if (k == 1) v.y = f; else if (k == 2) v.z = f; else v.w = f;
}

// Streaming 16-byte accesses: every byte is touched once per step, so the
// lines are marked evict-first (.cs), keeping L2 for the packed words and
// scales.  The load is a plain (non-volatile, no memory clobber) asm, so the
// compiler may issue a thread's later loads before its earlier stores; that
// is correct because no kernel here loads an address after the same thread
// stored to it (each element is read, then written once, the store
// depending on the load).
__device__ __forceinline__ float4 ld_stream(const float *p) {
    float4 v;
    asm("ld.global.cs.v4.f32 {%0, %1, %2, %3}, [%4];"
        : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
        : "l"(p));
    return v;
}
__device__ __forceinline__ void st_stream(float *p, const float4 &v) {
    asm volatile("st.global.cs.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z),
                 "f"(v.w));
}

// Asynchronous 16-byte global -> shared copies (sm_80+ LDGSTS), with an L2
// evict-first policy: the CTA queues the next workers' inputs while it
// computes on the current one.  Completion is awaited per thread with
// cp.async.wait_group (a hardware wait, no polling).
__device__ __forceinline__ uint64_t evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, uint64_t pol) {
    const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem),
                 "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// OR together the 4-bit groups of the 8 lanes that share one 32-bit sign
// word.  Lane l holds elements 4l..4l+3 of the warp's 128-element slot, so
// its nibble goes to bits 4*(l%8)..4*(l%8)+3 of word l/8.  Every lane of
// the group ends with the whole word.
__device__ __forceinline__ uint32_t gather_word(uint32_t nibble, int lane) {
    uint32_t v = nibble << (4 * (lane & 7));
    v |= __shfl_xor_sync(kFull, v, 1);
    v |= __shfl_xor_sync(kFull, v, 2);
    v |= __shfl_xor_sync(kFull, v, 4);
    return v;
}

// Element offset, within a tile, of slot u of a thread when each warp owns a
// contiguous span of kUnroll * 128 elements: warp `warp`'s slot u covers
// [512 warp + 128 u, +128), lane l holding elements 4l..4l+3 of it.  The
// warp's sign words for the span are then 4 * kUnroll consecutive words.
__device__ __forceinline__ int span_off(int warp, int lane, int u) {
    return (kUnroll * 128) * warp + 128 * u + 4 * lane;
}

// After gather_word for every slot, lanes 0, 8, 16, 24 hold words 4u..4u+3
// of slot u.  Bring word L of the warp's 4 * kUnroll to lane L so the warp
// stores all of them with one 64-byte, sector-aligned write.
__device__ __forceinline__ uint32_t collect_words(const uint32_t (&word)[kUnroll], int lane) {
    uint32_t mine = 0;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const uint32_t v = __shfl_sync(kFull, word[u], 8 * (lane & 3));
        if ((lane >> 2) == u) mine = v;
    }
    return mine;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}

// Fixed-order fp64 sum over a CTA of kScaleThreads threads (result valid in
// thread 0).
__device__ __forceinline__ double block_sum(double v, double *smem) {
    v = warp_sum(v);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) smem[warp] = v;
    __syncthreads();
    double acc = 0.0;
    if (threadIdx.x == 0)
        for (int k = 0; k < kScaleThreads / 32; ++k) acc += smem[k];
    return acc;
}

// Programmatic dependent launch (sm_90+).  A kernel launched with the
// programmatic-serialization attribute may start while the kernel before
// it on the stream is still finishing; grid_dependency_wait() blocks until
// every earlier grid of the stream has completed and its memory is visible,
// so each kernel calls it before reading anything an earlier kernel wrote.
// In a kernel launched without the attribute it returns at once.
// allow_dependent_launch() lets the next such kernel be scheduled once
// every CTA of this grid has called it (or exited); it has no effect on
// correctness, only on how early the next grid's CTAs are placed.
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
}
__device__ __forceinline__ void allow_dependent_launch() {
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

// The shard of the split step serving tile `tile_id`: the first q with
// tile_id < shard_end[q] (n_shards > 0; shard_end ascending, its last entry
// the number of tiles).
__device__ __forceinline__ int shard_of(int tile_id, int n_shards, const int *shard_end) {
    int q = 0;
    while (q < n_shards - 1 && tile_id >= shard_end[q]) ++q;
    return q;
}

// Real elements (0..4) of the float4 slot at tile offset off.
__device__ __forceinline__ int slot_real(int count, int off) { return min(4, max(0, count - off)); }

}  // namespace onebit
