// onebit.cu -- host side of libonebit: the C ABI declared in include/onebit.h.
//
// Owns host-side planning (padded layout, server chunks, the tile work
// list), argument and phase validation, workspace carving, kernel launches
// on the caller's stream, state read/write and the profiling counters.  It
// allocates no device memory: the caller passes the workspace.
//
// Method: "1-bit Adam: Communication Efficient Large-Scale Training with
// Adam's Convergence Speed" (review page), sections "Abstract" and
// "Proposed method" ([1BA]).
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <unordered_set>
#include <vector>

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>  // header-only; a no-op unless a profiler is attached

#include "../../include/onebit.h"
#include "onebit_kernels.cuh"

using onebit::Tile;
using onebit::kTile;
using onebit::kThreads;
using onebit::kScaleThreads;

namespace {

constexpr uint64_t kMagic = 0x31424954414441ull;  // "ADATIB1"
constexpr int64_t kMaxElements = int64_t(1) << 40;
constexpr int64_t kDecodeStage = int64_t(1) << 20;   // elements decoded per read round
constexpr int64_t kHostSlice = int64_t(1) << 22;     // gradient elements per worker per H2D slice
constexpr size_t kWsAlign = 256;

// ------------------------------------------------------------ test hook
std::mutex g_alloc_mu;
int g_fail_countdown = 0;

// Called before each host allocation; throws std::bad_alloc when the test
// hook's countdown reaches zero.
void host_alloc_point() {
    std::lock_guard<std::mutex> lk(g_alloc_mu);
    if (g_fail_countdown > 0 && --g_fail_countdown == 0) throw std::bad_alloc();
}

// ------------------------------------------------------ live contexts
std::mutex g_live_mu;
std::unordered_set<const ob_ctx *> g_live;

bool is_live(const ob_ctx *c) {
    std::lock_guard<std::mutex> lk(g_live_mu);
    return c && g_live.count(c) != 0;
}

// ------------------------------------------------------------ planning

int64_t round_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

// [1BA, Proposed method, 4]: server j of W owns sign words
// [j*cw, min(nw, (j+1)*cw)) of a tensor, cw = roundup(ceil(nw/W), 4).
void chunk_bounds(int64_t n, int W, int j, int64_t *b, int64_t *e) {
    const int64_t words = (n + 31) / 32;
    const int64_t per_server = round_up((words + W - 1) / W, 4);
    const int64_t lo = std::min<int64_t>(words, (int64_t)j * per_server);
    const int64_t hi = std::min<int64_t>(words, (int64_t)(j + 1) * per_server);
    *b = std::min<int64_t>(n, 32 * lo);
    *e = std::min<int64_t>(n, 32 * hi);
}

struct Plan {
    int T = 0, W = 0;
    std::vector<int64_t> numel, offset;
    int64_t n_pad = 0;
    std::vector<Tile> tiles;
    std::vector<int> tensor_tile_begin;  // [T+1]
    std::vector<int> chunk_tile_begin;   // [T*W+1]
    std::vector<int64_t> chunk_len;      // [T*W]
    // segmented scale reductions: first segment slot of each range, the
    // total number of slots, and the most segments of any range
    std::vector<int> tensor_seg_base, chunk_seg_base;
    int tensor_segs = 0, chunk_segs = 0, tensor_max_seg = 1, chunk_max_seg = 1;
};

int scale_segments(int tiles) {
    return tiles <= onebit::kScaleSegTiles ? 1
                                           : (tiles + onebit::kScaleSegTiles - 1) / onebit::kScaleSegTiles;
}

void plan_segments(const std::vector<int> &range_begin, std::vector<int> *base, int *total, int *most) {
    const size_t R = range_begin.size() - 1;
    base->assign(R, 0);
    int pos = 0;
    *most = 1;
    for (size_t r = 0; r < R; ++r) {
        const int nseg = scale_segments(range_begin[r + 1] - range_begin[r]);
        (*base)[r] = pos;
        pos += nseg;
        *most = std::max(*most, nseg);
    }
    *total = pos;
}

ob_status check_list(int n_tensors, const int64_t *numel) {
    if (n_tensors < 1 || !numel) return OB_ERR_INVALID_ARG;
    int64_t total = 0;
    for (int t = 0; t < n_tensors; ++t) {
        if (numel[t] < 0 || numel[t] > kMaxElements) return OB_ERR_INVALID_ARG;
        total += round_up(numel[t], OB_TENSOR_ALIGN);
        if (total > kMaxElements) return OB_ERR_INVALID_ARG;
    }
    return OB_OK;
}

// Padded layout, server chunks and the tile work list: tiles of up to kTile
// elements that never cross a tensor or chunk boundary, in layout order.
ob_status make_plan(int n_tensors, const int64_t *numel, int W, bool with_tiles, Plan *pl) {
    ob_status st = check_list(n_tensors, numel);
    if (st != OB_OK) return st;
    if (W < 1 || W > OB_MAX_WORKERS) return OB_ERR_INVALID_ARG;
    host_alloc_point();
    pl->T = n_tensors;
    pl->W = W;
    pl->numel.assign(numel, numel + n_tensors);
    pl->offset.resize(n_tensors);
    int64_t pos = 0;
    for (int t = 0; t < n_tensors; ++t) {
        pl->offset[t] = pos;
        pos += round_up(numel[t], OB_TENSOR_ALIGN);
    }
    pl->n_pad = pos;
    if (!with_tiles) return OB_OK;
    host_alloc_point();
    pl->tensor_tile_begin.assign(n_tensors + 1, 0);
    pl->chunk_tile_begin.assign((size_t)n_tensors * W + 1, 0);
    pl->chunk_len.assign((size_t)n_tensors * W, 0);
    int64_t count = 0;
    for (int t = 0; t < n_tensors; ++t) count += (numel[t] + kTile - 1) / kTile + W;
    if (count > INT32_MAX) return OB_ERR_INVALID_ARG;
    host_alloc_point();
    pl->tiles.reserve((size_t)count);
    for (int t = 0; t < n_tensors; ++t) {
        pl->tensor_tile_begin[t] = (int)pl->tiles.size();
        for (int j = 0; j < W; ++j) {
            const int c = t * W + j;
            pl->chunk_tile_begin[c] = (int)pl->tiles.size();
            int64_t b, e;
            chunk_bounds(numel[t], W, j, &b, &e);
            pl->chunk_len[c] = e - b;
            for (int64_t s = b; s < e; s += kTile) {
                Tile tl;
                tl.begin = pl->offset[t] + s;
                tl.count = (int32_t)std::min<int64_t>(kTile, e - s);
                tl.tensor = t;
                tl.chunk = j;
                tl.reserved = 0;
                pl->tiles.push_back(tl);
            }
        }
    }
    pl->tensor_tile_begin[n_tensors] = (int)pl->tiles.size();
    pl->chunk_tile_begin[(size_t)n_tensors * W] = (int)pl->tiles.size();
    host_alloc_point();
    plan_segments(pl->tensor_tile_begin, &pl->tensor_seg_base, &pl->tensor_segs, &pl->tensor_max_seg);
    plan_segments(pl->chunk_tile_begin, &pl->chunk_seg_base, &pl->chunk_segs, &pl->chunk_max_seg);
    return OB_OK;
}

// Byte offsets of the workspace regions.
struct Carve {
    size_t m, v, x, y, bits, sbits, s_prev, s_last, sp_prev, sp_last, partial_w, partial_s,
        counters_w, counters_s, seg_w, seg_s, tiles, tensor_tile_begin, chunk_tile_begin, numel,
        chunk_len, tensor_seg_base, chunk_seg_base, stage, ratio, pnorm, dnorm, partial_lamb,
        seg_lamb, counters_lamb, lamb_sums, total;
};

Carve carve(const Plan &pl) {
    Carve c{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = (off + bytes + kWsAlign - 1) / kWsAlign * kWsAlign;
        return o;
    };
    const size_t n = (size_t)pl.n_pad, W = (size_t)pl.W, T = (size_t)pl.T;
    const size_t nt = pl.tiles.size();
    c.m = take(n * 4);
    c.v = take(n * 4);
    c.x = take(W * n * 4);
    c.y = take(n * 4);
    c.bits = take(W * (n / 32) * 4);
    c.sbits = take((n / 32) * 4);
    c.s_prev = take(W * T * 4);
    c.s_last = take(W * T * 4);
    c.sp_prev = take(T * W * 4);
    c.sp_last = take(T * W * 4);
    c.partial_w = take(W * nt * 8);
    c.partial_s = take(nt * 8);
    c.counters_w = take(T * W * 4);
    c.counters_s = take(T * W * 4);
    c.seg_w = take((size_t)pl.tensor_segs * W * 8);
    c.seg_s = take((size_t)pl.chunk_segs * 8);
    c.tiles = take(nt * sizeof(Tile));
    c.tensor_tile_begin = take((T + 1) * 4);
    c.chunk_tile_begin = take((T * W + 1) * 4);
    c.numel = take(T * 8);
    c.chunk_len = take(T * W * 8);
    c.tensor_seg_base = take(T * 4);
    c.chunk_seg_base = take(T * W * 4);
    c.stage = take((size_t)kDecodeStage * 4);
    // 1-bit LAMB: trust ratios, ||p||^2 per tensor, D_j per chunk, and the
    // two-row reduction of the warmup's norms
    c.ratio = take(T * 4);
    c.pnorm = take(T * 8);
    c.dnorm = take(T * W * 8);
    c.partial_lamb = take(2 * nt * 8);
    c.seg_lamb = take(2 * (size_t)pl.tensor_segs * 8);
    c.counters_lamb = take(2 * T * 4);
    c.lamb_sums = take(2 * T * 8);
    c.total = off;
    return c;
}

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

// Runs of consecutive tiles whose padded span fits `limit` elements.
struct Run {
    int tile_lo, tile_hi;
    int64_t elem_lo, elem_hi;
};

std::vector<Run> make_runs(const std::vector<Tile> &tiles, int64_t limit) {
    host_alloc_point();
    std::vector<Run> runs;
    size_t k = 0;
    while (k < tiles.size()) {
        Run r;
        r.tile_lo = (int)k;
        r.elem_lo = tiles[k].begin;
        r.elem_hi = tiles[k].begin + round_up(tiles[k].count, OB_TENSOR_ALIGN);
        ++k;
        while (k < tiles.size()) {
            const int64_t hi = tiles[k].begin + round_up(tiles[k].count, OB_TENSOR_ALIGN);
            if (hi - r.elem_lo > limit) break;
            r.elem_hi = hi;
            ++k;
        }
        r.tile_hi = (int)k;
        runs.push_back(r);
    }
    return runs;
}

// Switches to a device for the duration of a call, then back.
struct DeviceGuard {
    int prev = -1;
    bool ok = true;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) {
            ok = false;
            return;
        }
        if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
    }
    ~DeviceGuard() {
        int cur;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

const char *const kKernelNames[OB_NUM_KERNELS] = {
    "ob_warmup_kernel", "ob_freeze_kernel",       "ob_pack_kernel", "ob_scale_kernel:worker",
    "ob_server_kernel", "ob_scale_kernel:server", "ob_apply_kernel"};

}  // namespace

// ------------------------------------------------------------------ ctx

// A compressed step recorded as a CUDA graph (graph mode).
struct StepGraph {
    bool built = false;
    bool lamb = false;           // built with the 1-bit LAMB update
    cudaGraph_t graph = nullptr;
    cudaGraphExec_t exec = nullptr;
    cudaGraphNode_t pack_node = nullptr, apply_node = nullptr;
    onebit::PackParams pack{};   // parameters last written into the nodes
    onebit::ApplyParams apply{};
    onebit::LambApplyParams lamb_apply{};
};

struct ob_ctx {
    uint64_t magic = kMagic;
    int device = 0;
    Plan plan;
    Carve cv;
    std::vector<Run> host_runs;
    float beta1, beta2, eps, lr, c1, c2;
    float *params = nullptr;
    char *ws = nullptr;
    cudaStream_t stream = nullptr;
    cudaStream_t copy_stream = nullptr;
    cudaEvent_t ev_copied[2] = {nullptr, nullptr};
    cudaEvent_t ev_consumed[2] = {nullptr, nullptr};
    cudaEvent_t ev_start = nullptr;
    int64_t t_warmup = 0, t_compressed = 0;
    bool frozen = false;
    // m is held densely in the m region (after create / warmup / a write),
    // or, after a compressed step, only as the server words and scales.
    bool m_dense = true;
    bool use_graph = true;  // graph mode (ob_graph_enable); used while the stream is not captured
    StepGraph graph;
    // 1-bit LAMB (ob_set_layerwise): layerwise trust ratios, recomputed every
    // step or (lamb_frozen) kept from the last warmup step; the norms the
    // compressed update needs are valid unless p or d changed otherwise
    bool lamb = false;
    bool lamb_frozen = false;
    bool pnorm_valid = false, dnorm_valid = false;
    bool broken = false;
    // split step: 0 idle, 1 after ob_worker_stage, 2 after ob_server_stage
    int split_stage = 0;
    // the server chunks this context serves in a split step: flat chunk
    // indices t * W + j in [chunk_lo, chunk_hi), contiguous in layout order
    // (ob_set_server_shard; all of them by default), shard `shard` of
    // n_shards
    int chunk_lo = 0, chunk_hi = -1;
    int n_shards = 1, shard = 0;
    // split step with peer memory (ob_set_peer_words): every shard's worker
    // rows and server words, as this process addresses them
    bool peer = false;
    std::vector<uint32_t *> peer_bits;
    std::vector<const uint32_t *> peer_sbits;
    // profiling
    bool profiling = false;
    std::vector<cudaEvent_t> event_pool;
    std::vector<std::pair<int, std::pair<cudaEvent_t, cudaEvent_t>>> pending;
    double kernel_ms[OB_NUM_KERNELS] = {};
    int64_t kernel_launches[OB_NUM_KERNELS] = {};

    template <class T> T *at(size_t off) const { return reinterpret_cast<T *>(ws + off); }
    float *m() const { return at<float>(cv.m); }
    float *v() const { return at<float>(cv.v); }
    float *x() const { return at<float>(cv.x); }
    float *y() const { return at<float>(cv.y); }
    uint32_t *bits() const { return at<uint32_t>(cv.bits); }
    uint32_t *sbits() const { return at<uint32_t>(cv.sbits); }
    float *s_prev() const { return at<float>(cv.s_prev); }
    float *s_last() const { return at<float>(cv.s_last); }
    float *sp_prev() const { return at<float>(cv.sp_prev); }
    float *sp_last() const { return at<float>(cv.sp_last); }
    double *partial_w() const { return at<double>(cv.partial_w); }
    double *partial_s() const { return at<double>(cv.partial_s); }
    Tile *tiles() const { return at<Tile>(cv.tiles); }
    int *tensor_tile_begin() const { return at<int>(cv.tensor_tile_begin); }
    int *chunk_tile_begin() const { return at<int>(cv.chunk_tile_begin); }
    int64_t *numel() const { return at<int64_t>(cv.numel); }
    int64_t *chunk_len() const { return at<int64_t>(cv.chunk_len); }
    unsigned *counters_w() const { return at<unsigned>(cv.counters_w); }
    unsigned *counters_s() const { return at<unsigned>(cv.counters_s); }
    double *seg_w() const { return at<double>(cv.seg_w); }
    double *seg_s() const { return at<double>(cv.seg_s); }
    int *tensor_seg_base() const { return at<int>(cv.tensor_seg_base); }
    int *chunk_seg_base() const { return at<int>(cv.chunk_seg_base); }
    float *stage() const { return at<float>(cv.stage); }
    float *ratio() const { return at<float>(cv.ratio); }
    double *pnorm() const { return at<double>(cv.pnorm); }
    double *dnorm() const { return at<double>(cv.dnorm); }
    double *partial_lamb() const { return at<double>(cv.partial_lamb); }
    double *seg_lamb() const { return at<double>(cv.seg_lamb); }
    unsigned *counters_lamb() const { return at<unsigned>(cv.counters_lamb); }
    double *lamb_sums() const { return at<double>(cv.lamb_sums); }
    int n_tiles() const { return (int)plan.tiles.size(); }
};

namespace {

ob_status fail_cuda(ob_ctx *c, cudaError_t e) {
    if (e == cudaSuccess) return OB_OK;
    if (c) c->broken = true;
    return OB_ERR_CUDA;
}

ob_status check_ctx(const ob_ctx *c) {
    if (!is_live(c) || c->magic != kMagic) return OB_ERR_INVALID_ARG;
    if (c->broken) return OB_ERR_CUDA;
    return OB_OK;
}

// Profiling: an event pair around one kernel, summed at ob_profile_read.
cudaEvent_t take_event(ob_ctx *c) {
    if (!c->event_pool.empty()) {
        cudaEvent_t e = c->event_pool.back();
        c->event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

// An NVTX range over one library call (shown by Nsight tools beside the
// CUDA launches it makes).
struct NvtxCall {
    explicit NvtxCall(const char *name) { nvtxRangePushA(name); }
    ~NvtxCall() { nvtxRangePop(); }
    NvtxCall(const NvtxCall &) = delete;
    NvtxCall &operator=(const NvtxCall &) = delete;
};

// Around each kernel launch: an NVTX range named after the kernel and,
// while profiling is on, a pair of CUDA events on the context's stream.
struct KernelTimer {
    ob_ctx *c;
    int id;
    cudaEvent_t a = nullptr, b = nullptr;
    nvtxRangeId_t range = 0;
    KernelTimer(ob_ctx *ctx, int k) : c(ctx), id(k) {
        range = nvtxRangeStartA(kKernelNames[k]);
        if (!c->profiling) return;
        a = take_event(c);
        b = take_event(c);
        if (a && b) {
            cudaEventRecord(a, c->stream);
        } else {  // no timing for this launch; keep whichever event was made
            if (a) c->event_pool.push_back(a);
            if (b) c->event_pool.push_back(b);
            a = b = nullptr;
        }
    }
    void stop() {
        if (range) nvtxRangeEnd(range);
        range = 0;
        if (!c->profiling || !a || !b) return;
        cudaEventRecord(b, c->stream);
        c->pending.push_back({id, {a, b}});
        a = b = nullptr;
    }
};

dim3 grid1(int n) { return dim3((unsigned)n); }

// ---------------------------------------------------------------- launches
//
// The five launches of a compressed step (worker stage, worker scales,
// server stage, server scales, update), each with its parameters built by
// one function, so direct launches and the CUDA-graph nodes of graph mode
// are the same launches.

// Range sums of per-tile partial sums (ob_scale_kernel): the worker and
// server scales, and plain sums for 1-bit LAMB's norms.  Worker scales:
// ranges = tensors, one row per worker, scale (t, w) at s_prev[w * T + t].
onebit::ScaleParams worker_scale_params(const ob_ctx *c) {
    onebit::ScaleParams P{};  // zeroed, padding too: compared bytewise in graph mode
    P.partial = c->partial_w();
    P.n_tiles = c->n_tiles();
    P.range_begin = c->tensor_tile_begin();
    P.seg_base = c->tensor_seg_base();
    P.count = c->numel();
    P.seg = c->seg_w();
    P.counter = c->counters_w();
    P.out_prev = c->s_prev();
    P.out_last = c->s_last();
    P.rows = c->plan.W;
    P.R = c->plan.T;
    P.out_stride_r = 1;
    P.out_stride_row = c->plan.T;
    return P;
}

onebit::ScaleParams server_scale_params(const ob_ctx *c) {
    onebit::ScaleParams P{};  // zeroed, padding too: compared bytewise in graph mode
    P.partial = c->partial_s();
    P.n_tiles = c->n_tiles();
    P.range_begin = c->chunk_tile_begin();
    P.seg_base = c->chunk_seg_base();
    P.count = c->chunk_len();
    P.seg = c->seg_s();
    P.counter = c->counters_s();
    P.out_prev = c->sp_prev();
    P.out_last = c->sp_last();
    P.rows = 1;
    P.R = c->plan.T * c->plan.W;
    P.out_stride_r = 1;
    P.out_stride_row = 0;
    return P;
}

// Plain sums per tensor of `rows` rows of per-tile partials (rows <= 2):
// out[row * T + t].  Uses the worker scales' buffers for one row and the
// 1-bit LAMB ones for two.
onebit::ScaleParams tensor_sum_params(const ob_ctx *c, const double *partial, int rows, double *out) {
    onebit::ScaleParams P{};  // zeroed, padding too: compared bytewise in graph mode
    P.partial = partial;
    P.n_tiles = c->n_tiles();
    P.range_begin = c->tensor_tile_begin();
    P.seg_base = c->tensor_seg_base();
    P.count = c->numel();
    P.seg = rows == 1 ? c->seg_w() : c->seg_lamb();
    P.counter = rows == 1 ? c->counters_w() : c->counters_lamb();
    P.out_sum = out;
    P.rows = rows;
    P.R = c->plan.T;
    P.out_stride_r = 1;
    P.out_stride_row = c->plan.T;
    return P;
}

// Plain sums per server chunk of one row of per-tile partials: out[t * W + j].
onebit::ScaleParams chunk_sum_params(const ob_ctx *c, const double *partial, double *out) {
    onebit::ScaleParams P = server_scale_params(c);
    P.partial = partial;
    P.out_prev = P.out_last = nullptr;
    P.out_sum = out;
    return P;
}

onebit::PackParams pack_params(const ob_ctx *c, const float *const *g, int64_t g_offset,
                               int tile_lo) {
    onebit::PackParams P{};  // zeroed, padding too: compared bytewise in graph mode
    P.tiles = c->tiles();
    P.tile_base = tile_lo;
    P.n_tiles = c->n_tiles();
    P.m = c->m();
    P.m_bits = c->sbits();
    P.m_scale = c->sp_last();
    P.m_dense = c->m_dense ? 1 : 0;
    P.chunks = c->plan.W;
    for (int w = 0; w < OB_MAX_WORKERS; ++w) P.g[w] = w < c->plan.W ? g[w] : nullptr;
    P.g_offset = g_offset;
    P.x = c->x();
    P.bits = c->bits();
    P.s_prev = c->s_prev();
    P.partial = c->partial_w();
    P.n_pad = c->plan.n_pad;
    P.W = c->plan.W;
    P.T = c->plan.T;
    P.beta1 = c->beta1;
    P.c1 = c->c1;
    return P;
}

onebit::ServerParams server_params(const ob_ctx *c) {
    const int W = c->plan.W;
    onebit::ServerParams P{};  // zeroed, padding too: compared bytewise in graph mode
    P.tiles = c->tiles();
    P.bits = c->bits();
    P.s_w = c->s_prev();
    P.y = c->y();
    P.sp_prev = c->sp_prev();
    P.sbits = c->sbits();
    P.partial = c->partial_s();
    P.n_pad = c->plan.n_pad;
    P.W = W;
    P.T = c->plan.T;
    P.w_pow2 = (W & (W - 1)) == 0;
    P.inv_w = 1.0f / (float)W;  // exact for a power of two
    return P;
}

onebit::ApplyParams apply_params(const ob_ctx *c) {
    onebit::ApplyParams P{};  // zeroed, padding too: compared bytewise in graph mode
    P.tiles = c->tiles();
    P.sbits = c->sbits();
    P.sp = c->sp_last();
    P.d = c->v();
    P.p = c->params;
    P.m = nullptr;  // m stays as (sbits, sp_last); see ob_ctx::m_dense
    P.W = c->plan.W;
    P.lr = c->lr;
    return P;
}

// The 1-bit LAMB update: apply_params with the layerwise rates; its
// per-tile sums of the new p^2 go to the worker stage's partial-sum row 0
// (free once the worker scales are done) and are reduced per tensor into
// pnorm by a range-sum launch after it.
onebit::LambApplyParams lamb_apply_params(const ob_ctx *c) {
    onebit::LambApplyParams P{};  // zeroed, padding too: compared bytewise in graph mode
    P.a = apply_params(c);
    P.tensor_tile_begin = c->tensor_tile_begin();
    P.pnorm = c->pnorm();
    P.dnorm = c->dnorm();
    P.ratio = c->ratio();
    P.partial = c->partial_w();
    P.fixed_ratio = c->lamb_frozen ? 1 : 0;
    return P;
}

// Launch geometry of each kernel: grid, block, dynamic shared memory.
struct Geometry {
    dim3 grid, block;
    size_t smem;
};
Geometry pack_geometry(int tiles) { return {grid1(tiles), dim3(kThreads), (size_t)onebit::kPackSmemBytes}; }
Geometry range_sum_geometry(int ranges, int rows, int max_seg) {
    return {dim3((unsigned)ranges, (unsigned)rows, (unsigned)max_seg), dim3(kScaleThreads), 0};
}
Geometry worker_scale_geometry(const ob_ctx *c) {
    return range_sum_geometry(c->plan.T, c->plan.W, c->plan.tensor_max_seg);
}
Geometry server_geometry(int tiles, int W) {
    return {grid1(tiles), dim3(kThreads), (size_t)W * onebit::kTileWords * sizeof(uint32_t)};
}
Geometry server_scale_geometry(const ob_ctx *c) {
    return range_sum_geometry(c->plan.T * c->plan.W, 1, c->plan.chunk_max_seg);
}
Geometry apply_geometry(const ob_ctx *c) { return {grid1(c->n_tiles()), dim3(kThreads), 0}; }

// One kernel launch on the context's stream, allowed to start while the
// stream's previous kernel finishes (programmatic dependent launch: every
// kernel of the step waits for its predecessors' results inside, with
// grid_dependency_wait, before it reads them).  Returns this launch's own
// status.
template <class Params>
cudaError_t launch(void (*kernel)(Params), const Geometry &G, const Params &P, cudaStream_t stream) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = G.grid;
    cfg.blockDim = G.block;
    cfg.dynamicSmemBytes = G.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, P);
}

ob_status launch_pack(ob_ctx *c, const float *const *g, int64_t g_offset, int tile_lo, int tile_hi) {
    if (tile_hi <= tile_lo) return OB_OK;
    const onebit::PackParams P = pack_params(c, g, g_offset, tile_lo);
    return fail_cuda(c, launch(onebit::ob_pack_kernel, pack_geometry(tile_hi - tile_lo), P, c->stream));
}

int shard_tile_end(const Plan &pl, int G, int q);

// In the split step with peer memory, the update reads each chunk's server
// words from the process serving it and copies them into this context's.
void add_peer_sources(const ob_ctx *c, onebit::ApplyParams *A) {
    if (!c->peer || c->split_stage != 2) return;
    A->n_shards = c->n_shards;
    for (int q = 0; q < c->n_shards; ++q) {
        A->shard_end[q] = shard_tile_end(c->plan, c->n_shards, q);
        A->src_sbits[q] = c->peer_sbits[q];
    }
    A->sbits_copy = c->sbits();
}

// The gather and update (1-bit LAMB's with layerwise rates when on; then
// its new ||p||^2 summed per tensor for the next step).
ob_status launch_apply(ob_ctx *c) {
    if (c->n_tiles() == 0) return OB_OK;
    KernelTimer k(c, OB_K_APPLY);
    cudaError_t e;
    if (c->lamb) {
        onebit::LambApplyParams L = lamb_apply_params(c);
        add_peer_sources(c, &L.a);
        e = launch(onebit::ob_lamb_apply_kernel, apply_geometry(c), L, c->stream);
    } else {
        onebit::ApplyParams A = apply_params(c);
        add_peer_sources(c, &A);
        e = launch(onebit::ob_apply_kernel, apply_geometry(c), A, c->stream);
    }
    if (e == cudaSuccess && c->lamb && !c->lamb_frozen)
        e = launch(onebit::ob_scale_kernel, range_sum_geometry(c->plan.T, 1, c->plan.tensor_max_seg),
                   tensor_sum_params(c, c->partial_w(), 1, c->pnorm()), c->stream);
    k.stop();
    return fail_cuda(c, e);
}

// 1-bit LAMB: recompute D_j (want_d) and ||p||^2 (want_p) from d and p.
ob_status launch_lamb_norms(ob_ctx *c, bool want_d, bool want_p) {
    if (!want_d && !want_p) return OB_OK;
    if (c->n_tiles() > 0) {
        onebit::LambNormsParams P{};
        P.tiles = c->tiles();
        P.d = c->v();
        P.p = c->params;
        P.partial_d = c->partial_s();
        P.partial_p = c->partial_w();
        P.want_d = want_d ? 1 : 0;
        P.want_p = want_p ? 1 : 0;
        KernelTimer k(c, OB_K_FREEZE);
        cudaError_t e = launch(onebit::ob_lamb_norms_kernel, Geometry{grid1(c->n_tiles()), dim3(kThreads), 0},
                               P, c->stream);
        if (e == cudaSuccess && want_d)
            e = launch(onebit::ob_scale_kernel, server_scale_geometry(c),
                       chunk_sum_params(c, c->partial_s(), c->dnorm()), c->stream);
        if (e == cudaSuccess && want_p)
            e = launch(onebit::ob_scale_kernel, range_sum_geometry(c->plan.T, 1, c->plan.tensor_max_seg),
                       tensor_sum_params(c, c->partial_w(), 1, c->pnorm()), c->stream);
        k.stop();
        ob_status st = fail_cuda(c, e);
        if (st != OB_OK) return st;
    }
    if (want_d) c->dnorm_valid = true;
    if (want_p) c->pnorm_valid = true;
    return OB_OK;
}

// Before a 1-bit LAMB compressed step: the norms its update reads.
ob_status ensure_lamb_norms(ob_ctx *c) {
    if (!c->lamb || c->lamb_frozen) return OB_OK;  // kept ratios need no norms
    return launch_lamb_norms(c, !c->dnorm_valid, !c->pnorm_valid);
}

// Everything of a compressed step after the worker stage's tile kernels:
// the worker scales, the server stage, the server scales, the update.
ob_status launch_after_pack(ob_ctx *c, KernelTimer &pack_timer) {
    const int nt = c->n_tiles();
    pack_timer.stop();
    {
        KernelTimer k(c, OB_K_PACK_SCALE);
        const cudaError_t e =
            launch(onebit::ob_scale_kernel, worker_scale_geometry(c), worker_scale_params(c), c->stream);
        k.stop();
        ob_status st = fail_cuda(c, e);
        if (st != OB_OK) return st;
    }
    if (nt > 0) {
        KernelTimer k(c, OB_K_SERVER);
        const cudaError_t e =
            launch(onebit::ob_server_kernel, server_geometry(nt, c->plan.W), server_params(c), c->stream);
        k.stop();
        ob_status st = fail_cuda(c, e);
        if (st != OB_OK) return st;
    }
    {
        KernelTimer k(c, OB_K_SERVER_SCALE);
        const cudaError_t e =
            launch(onebit::ob_scale_kernel, server_scale_geometry(c), server_scale_params(c), c->stream);
        k.stop();
        ob_status st = fail_cuda(c, e);
        if (st != OB_OK) return st;
    }
    return launch_apply(c);
}

// ------------------------------------------------------------- graph mode
//
// The step's kernels as one CUDA graph: a chain of kernel nodes built once
// (lazily), replayed with one launch.  Parameters that change between
// steps (gradient pointers, dense or lazy momentum, the learning rate) are
// written into the instantiated graph's nodes before the replay.

template <class Params>
cudaKernelNodeParams node_params(void *func, const Geometry &G, Params *P, void **args) {
    cudaKernelNodeParams kp{};
    kp.func = func;
    kp.gridDim = G.grid;
    kp.blockDim = G.block;
    kp.sharedMemBytes = (unsigned)G.smem;
    args[0] = P;
    kp.kernelParams = args;
    kp.extra = nullptr;
    return kp;
}

void destroy_graph(ob_ctx *c);

ob_status build_graph(ob_ctx *c, const float *const *g) {
    StepGraph &sg = c->graph;
    cudaError_t e = cudaGraphCreate(&sg.graph, 0);
    cudaGraphNode_t prev = nullptr;
    auto add = [&](void *func, const Geometry &G, auto *P, cudaGraphNode_t *out) {
        if (e != cudaSuccess) return;
        void *args[1];
        const cudaKernelNodeParams kp = node_params(func, G, P, args);
        e = cudaGraphAddKernelNode(out, sg.graph, prev ? &prev : nullptr, prev ? 1 : 0, &kp);
        if (e == cudaSuccess) prev = *out;
    };
    const int nt = c->n_tiles();
    sg.pack = pack_params(c, g, 0, 0);
    sg.apply = apply_params(c);
    sg.lamb_apply = lamb_apply_params(c);
    sg.lamb = c->lamb;
    onebit::ServerParams sv = server_params(c);
    onebit::ScaleParams ws = worker_scale_params(c), ss = server_scale_params(c);
    onebit::ScaleParams pn = tensor_sum_params(c, c->partial_w(), 1, c->pnorm());
    cudaGraphNode_t n_ws, n_sv, n_ss, n_pn;
    if (nt > 0) add((void *)onebit::ob_pack_kernel, pack_geometry(nt), &sg.pack, &sg.pack_node);
    add((void *)onebit::ob_scale_kernel, worker_scale_geometry(c), &ws, &n_ws);
    if (nt > 0) add((void *)onebit::ob_server_kernel, server_geometry(nt, c->plan.W), &sv, &n_sv);
    add((void *)onebit::ob_scale_kernel, server_scale_geometry(c), &ss, &n_ss);
    if (nt > 0) {
        if (sg.lamb) {
            add((void *)onebit::ob_lamb_apply_kernel, apply_geometry(c), &sg.lamb_apply, &sg.apply_node);
            if (!c->lamb_frozen)
                add((void *)onebit::ob_scale_kernel, range_sum_geometry(c->plan.T, 1, c->plan.tensor_max_seg),
                    &pn, &n_pn);
        } else {
            add((void *)onebit::ob_apply_kernel, apply_geometry(c), &sg.apply, &sg.apply_node);
        }
    }
    if (e == cudaSuccess) e = cudaGraphInstantiate(&sg.exec, sg.graph, 0);
    if (e != cudaSuccess) {
        destroy_graph(c);
        return fail_cuda(c, e);
    }
    sg.built = true;
    return OB_OK;
}

void destroy_graph(ob_ctx *c) {
    StepGraph &sg = c->graph;
    if (sg.exec) cudaGraphExecDestroy(sg.exec);
    if (sg.graph) cudaGraphDestroy(sg.graph);
    sg = StepGraph{};
}

// One compressed step through the graph.
ob_status graph_step(ob_ctx *c, const float *const *g) {
    StepGraph &sg = c->graph;
    if (!sg.built) {
        ob_status st = build_graph(c, g);
        if (st != OB_OK) return st;
    }
    const int nt = c->n_tiles();
    cudaError_t e = cudaSuccess;
    if (nt > 0) {
        onebit::PackParams P = pack_params(c, g, 0, 0);
        if (std::memcmp(&P, &sg.pack, sizeof P) != 0) {
            sg.pack = P;
            void *args[1];
            const cudaKernelNodeParams kp =
                node_params((void *)onebit::ob_pack_kernel, pack_geometry(nt), &sg.pack, args);
            e = cudaGraphExecKernelNodeSetParams(sg.exec, sg.pack_node, &kp);
        }
        if (sg.lamb) {
            onebit::LambApplyParams A = lamb_apply_params(c);
            if (e == cudaSuccess && std::memcmp(&A, &sg.lamb_apply, sizeof A) != 0) {
                sg.lamb_apply = A;
                void *args[1];
                const cudaKernelNodeParams kp = node_params((void *)onebit::ob_lamb_apply_kernel,
                                                            apply_geometry(c), &sg.lamb_apply, args);
                e = cudaGraphExecKernelNodeSetParams(sg.exec, sg.apply_node, &kp);
            }
        } else {
            onebit::ApplyParams A = apply_params(c);
            if (e == cudaSuccess && std::memcmp(&A, &sg.apply, sizeof A) != 0) {
                sg.apply = A;
                void *args[1];
                const cudaKernelNodeParams kp =
                    node_params((void *)onebit::ob_apply_kernel, apply_geometry(c), &sg.apply, args);
                e = cudaGraphExecKernelNodeSetParams(sg.exec, sg.apply_node, &kp);
            }
        }
    }
    if (e == cudaSuccess) e = cudaGraphLaunch(sg.exec, c->stream);
    return fail_cuda(c, e);
}

ob_status check_grads(const ob_ctx *c, const float *const *g) {
    if (!g) return OB_ERR_INVALID_ARG;
    if (c->plan.n_pad == 0) return OB_OK;  // nothing is read
    for (int w = 0; w < c->plan.W; ++w) {
        if (!g[w]) return OB_ERR_INVALID_ARG;
        if (!aligned(g[w], 16)) return OB_ERR_ALIGN;
    }
    return OB_OK;
}

size_t state_bytes(const ob_ctx *c, int kind) {
    const size_t n = (size_t)c->plan.n_pad, W = (size_t)c->plan.W, T = (size_t)c->plan.T;
    switch (kind) {
    case OB_STATE_P: case OB_STATE_M: case OB_STATE_V: case OB_STATE_D:
    case OB_STATE_E_WORKER: case OB_STATE_E_SERVER:
        return n * 4;
    case OB_STATE_S_WORKER: case OB_STATE_S_SERVER:
        return W * T * 4;
    case OB_STATE_BITS_WORKER: case OB_STATE_BITS_SERVER:
        return (n / 32) * 4;
    case OB_STATE_STEP:
        return 3 * sizeof(int64_t);
    case OB_STATE_RATIO:
        return T * 4;
    default:
        return 0;
    }
}

// Decode a lazily stored buffer into host memory, run by run through the
// staging region.  launch(run, out, out_base) queues the decoder of one run.
template <class Launch>
ob_status read_decoded(ob_ctx *c, float *host, Launch launch) {
    std::memset(host, 0, (size_t)c->plan.n_pad * 4);
    std::vector<Run> runs = make_runs(c->plan.tiles, kDecodeStage);
    for (const Run &r : runs) {
        const int64_t span = r.elem_hi - r.elem_lo;
        ob_status st = fail_cuda(c, cudaMemsetAsync(c->stage(), 0, (size_t)span * 4, c->stream));
        if (st != OB_OK) return st;
        launch(r, c->stage(), r.elem_lo);
        st = fail_cuda(c, cudaGetLastError());
        if (st != OB_OK) return st;
        st = fail_cuda(c, cudaMemcpyAsync(host + r.elem_lo, c->stage(), (size_t)span * 4,
                                          cudaMemcpyDeviceToHost, c->stream));
        if (st != OB_OK) return st;
        st = fail_cuda(c, cudaStreamSynchronize(c->stream));
        if (st != OB_OK) return st;
    }
    return OB_OK;
}

// Error buffer (x or y with its scales): e = fl(x - sign(x) s).
ob_status read_error(ob_ctx *c, const float *src, const float *scales, int stride_t, int stride_j,
                     float *host) {
    return read_decoded(c, host, [&](const Run &r, float *out, int64_t base) {
        onebit::DecodeParams P;
        P.tiles = c->tiles();
        P.tile_base = r.tile_lo;
        P.x = src;
        P.scales = scales;
        P.stride_t = stride_t;
        P.stride_j = stride_j;
        P.out = out;
        P.out_base = base;
        onebit::ob_decode_error_kernel<<<grid1(r.tile_hi - r.tile_lo), kThreads, 0, c->stream>>>(P);
    });
}

// Momentum held as server words and scales: m = sign' s'_j.
void launch_decode_momentum(ob_ctx *c, int tile_lo, int tile_hi, float *out, int64_t base) {
    onebit::ob_decode_momentum_kernel<<<grid1(tile_hi - tile_lo), kThreads, 0, c->stream>>>(
        c->tiles(), tile_lo, c->sbits(), c->sp_last(), c->plan.W, out, base);
}

// Chunks [*lo, *hi) of shard r of G: contiguous in (tensor, chunk) order,
// cut where the running tile count reaches r/G of all tiles, so every
// shard gets about the same server-stage work.
void shard_chunks(const Plan &pl, int G, int r, int *lo, int *hi) {
    const int C = pl.T * pl.W;
    const int64_t nt = (int64_t)pl.tiles.size();
    auto cut = [&](int q) {
        if (q <= 0) return 0;
        if (q >= G) return C;
        const int64_t target = nt * q / G;
        return (int)(std::lower_bound(pl.chunk_tile_begin.begin(), pl.chunk_tile_begin.begin() + C + 1,
                                      target) - pl.chunk_tile_begin.begin());
    };
    *lo = cut(r);
    *hi = cut(r + 1);
}

// One past the last tile of shard q of G (the tiles of its chunks).
int shard_tile_end(const Plan &pl, int G, int q) {
    int lo, hi;
    shard_chunks(pl, G, q, &lo, &hi);
    return pl.chunk_tile_begin[hi];
}

// First server word of flat chunk c (n_pad/32 for c == T*W): chunk j of a
// tensor starts at word min(nw, j*cw) of the tensor.
int64_t chunk_first_word(const Plan &pl, int c) {
    if (c >= pl.T * pl.W) return pl.n_pad / 32;
    const int t = c / pl.W, j = c % pl.W;
    const int64_t nw = (pl.numel[t] + 31) / 32;
    const int64_t cw = round_up((nw + pl.W - 1) / pl.W, 4);
    return pl.offset[t] / 32 + std::min<int64_t>(nw, (int64_t)j * cw);
}

// Rebuild the dense momentum in its own region (before a consumer that
// needs it dense: the warmup step).
ob_status materialize_momentum(ob_ctx *c) {
    if (c->m_dense) return OB_OK;
    if (c->n_tiles() > 0) {
        launch_decode_momentum(c, 0, c->n_tiles(), c->m(), 0);
        ob_status st = fail_cuda(c, cudaGetLastError());
        if (st != OB_OK) return st;
    }
    c->m_dense = true;
    return OB_OK;
}

}  // namespace

// ================================================================= C ABI

extern "C" {

const char *ob_status_string(ob_status s) {
    switch (s) {
    case OB_OK: return "OB_OK";
    case OB_ERR_INVALID_ARG: return "OB_ERR_INVALID_ARG";
    case OB_ERR_PHASE: return "OB_ERR_PHASE";
    case OB_ERR_ALIGN: return "OB_ERR_ALIGN";
    case OB_ERR_WORKSPACE: return "OB_ERR_WORKSPACE";
    case OB_ERR_OOM: return "OB_ERR_OOM";
    case OB_ERR_CUDA: return "OB_ERR_CUDA";
    case OB_ERR_DEVICE_TIMEOUT: return "OB_ERR_DEVICE_TIMEOUT";
    }
    return "OB_UNKNOWN_STATUS";
}

int ob_abi_version(void) { return OB_ABI_VERSION; }

const char *ob_kernel_name(int id) {
    return (id >= 0 && id < OB_NUM_KERNELS) ? kKernelNames[id] : nullptr;
}

void ob_test_fail_host_alloc(int countdown) {
    std::lock_guard<std::mutex> lk(g_alloc_mu);
    g_fail_countdown = countdown > 0 ? countdown : 0;
}

ob_status ob_layout(int n_tensors, const int64_t *numel, int64_t *tensor_offsets,
                    int64_t *n_padded) {
    if (!n_padded) return OB_ERR_INVALID_ARG;
    ob_status st = check_list(n_tensors, numel);
    if (st != OB_OK) return st;
    int64_t pos = 0;
    for (int t = 0; t < n_tensors; ++t) {
        if (tensor_offsets) tensor_offsets[t] = pos;
        pos += round_up(numel[t], OB_TENSOR_ALIGN);
    }
    *n_padded = pos;
    return OB_OK;
}

ob_status ob_chunk_range(int64_t numel, int W, int j, int64_t *begin, int64_t *end) {
    if (numel < 0 || W < 1 || W > OB_MAX_WORKERS || j < 0 || j >= W || !begin || !end)
        return OB_ERR_INVALID_ARG;
    chunk_bounds(numel, W, j, begin, end);
    return OB_OK;
}

ob_status ob_workspace_bytes(int n_tensors, const int64_t *numel, int W, size_t *bytes) {
    if (!bytes) return OB_ERR_INVALID_ARG;
    try {
        Plan pl;
        ob_status st = make_plan(n_tensors, numel, W, true, &pl);
        if (st != OB_OK) return st;
        *bytes = carve(pl).total;
        return OB_OK;
    } catch (const std::bad_alloc &) {
        return OB_ERR_OOM;
    }
}

ob_status ob_create(int n_tensors, const int64_t *numel, int W, float beta1, float beta2,
                    float eps, float lr, float *d_params, void *d_workspace,
                    size_t workspace_bytes, void *cuda_stream, ob_ctx **out) {
    if (!out) return OB_ERR_INVALID_ARG;
    *out = nullptr;
    if (!d_workspace) return OB_ERR_INVALID_ARG;
    if (!(beta1 >= 0.f && beta1 < 1.f) || !(beta2 >= 0.f && beta2 < 1.f) || !(eps > 0.f) ||
        !std::isfinite(lr) || !std::isfinite(eps))
        return OB_ERR_INVALID_ARG;
    if (!aligned(d_params, 16) || !aligned(d_workspace, kWsAlign)) return OB_ERR_ALIGN;
    ob_ctx *c = nullptr;
    try {
        host_alloc_point();
        c = new ob_ctx();
        ob_status st = make_plan(n_tensors, numel, W, true, &c->plan);
        if (st != OB_OK) {
            delete c;
            return st;
        }
        if (!d_params && c->plan.n_pad > 0) {  // NULL only for an all-empty list
            delete c;
            return OB_ERR_INVALID_ARG;
        }
        c->cv = carve(c->plan);
        if (workspace_bytes < c->cv.total) {
            delete c;
            return OB_ERR_WORKSPACE;
        }
        c->host_runs = make_runs(c->plan.tiles, kHostSlice);
    } catch (const std::bad_alloc &) {
        delete c;
        return OB_ERR_OOM;
    }
    c->beta1 = beta1;
    c->beta2 = beta2;
    c->eps = eps;
    c->lr = lr;
    c->c1 = 1.0f - beta1;
    c->c2 = 1.0f - beta2;
    c->params = d_params;
    c->ws = static_cast<char *>(d_workspace);
    c->stream = static_cast<cudaStream_t>(cuda_stream);
    // Release what was created so far and report `status`.
    auto bail = [&](ob_status status) {
        if (c->copy_stream) cudaStreamDestroy(c->copy_stream);
        for (auto &ev : c->ev_copied) if (ev) cudaEventDestroy(ev);
        for (auto &ev : c->ev_consumed) if (ev) cudaEventDestroy(ev);
        if (c->ev_start) cudaEventDestroy(c->ev_start);
        delete c;
        return status;
    };
    cudaError_t e = cudaGetDevice(&c->device);
    if (e != cudaSuccess) return bail(OB_ERR_CUDA);
    e = cudaFuncSetAttribute(onebit::ob_pack_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             onebit::kPackSmemBytes);
    if (e != cudaSuccess) return bail(OB_ERR_CUDA);
    e = cudaStreamCreateWithFlags(&c->copy_stream, cudaStreamNonBlocking);
    if (e != cudaSuccess) return bail(OB_ERR_CUDA);
    for (int k = 0; k < 2 && e == cudaSuccess; ++k) {
        e = cudaEventCreateWithFlags(&c->ev_copied[k], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->ev_consumed[k], cudaEventDisableTiming);
    }
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->ev_start, cudaEventDisableTiming);
    if (e != cudaSuccess) return bail(OB_ERR_CUDA);
    // zero the state, upload the work list
    const Plan &pl = c->plan;
    e = cudaMemsetAsync(c->ws, 0, c->cv.tiles, c->stream);
    if (e == cudaSuccess && !pl.tiles.empty())
        e = cudaMemcpyAsync(c->tiles(), pl.tiles.data(), pl.tiles.size() * sizeof(Tile),
                            cudaMemcpyHostToDevice, c->stream);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(c->tensor_tile_begin(), pl.tensor_tile_begin.data(),
                            pl.tensor_tile_begin.size() * 4, cudaMemcpyHostToDevice, c->stream);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(c->chunk_tile_begin(), pl.chunk_tile_begin.data(),
                            pl.chunk_tile_begin.size() * 4, cudaMemcpyHostToDevice, c->stream);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(c->numel(), pl.numel.data(), pl.numel.size() * 8, cudaMemcpyHostToDevice,
                            c->stream);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(c->chunk_len(), pl.chunk_len.data(), pl.chunk_len.size() * 8,
                            cudaMemcpyHostToDevice, c->stream);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(c->tensor_seg_base(), pl.tensor_seg_base.data(),
                            pl.tensor_seg_base.size() * 4, cudaMemcpyHostToDevice, c->stream);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(c->chunk_seg_base(), pl.chunk_seg_base.data(),
                            pl.chunk_seg_base.size() * 4, cudaMemcpyHostToDevice, c->stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(c->stream);
    if (e != cudaSuccess) return bail(OB_ERR_CUDA);
    {
        std::lock_guard<std::mutex> lk(g_live_mu);
        try {
            g_live.insert(c);
        } catch (const std::bad_alloc &) {
            return bail(OB_ERR_OOM);
        }
    }
    *out = c;
    return OB_OK;
}

void ob_destroy(ob_ctx *c) {
    {
        std::lock_guard<std::mutex> lk(g_live_mu);
        if (!c || g_live.erase(c) == 0) return;
    }
    DeviceGuard dg(c->device);
    cudaStreamSynchronize(c->stream);
    cudaStreamSynchronize(c->copy_stream);
    for (auto &p : c->pending) {
        cudaEventDestroy(p.second.first);
        cudaEventDestroy(p.second.second);
    }
    for (cudaEvent_t e : c->event_pool) cudaEventDestroy(e);
    for (auto &ev : c->ev_copied) cudaEventDestroy(ev);
    for (auto &ev : c->ev_consumed) cudaEventDestroy(ev);
    cudaEventDestroy(c->ev_start);
    cudaStreamDestroy(c->copy_stream);
    destroy_graph(c);
    c->magic = 0;
    delete c;
}

ob_status ob_warmup_adam_step(ob_ctx *c, const float *const *d_grads) {
    NvtxCall nvtx("ob_warmup_adam_step");
    ob_status st = check_ctx(c);
    if (st != OB_OK) return st;
    if (c->frozen || c->split_stage != 0) return OB_ERR_PHASE;
    if ((st = check_grads(c, d_grads)) != OB_OK) return st;
    DeviceGuard dg(c->device);
    if (!dg.ok) return fail_cuda(c, cudaErrorInvalidDevice);
    if ((st = materialize_momentum(c)) != OB_OK) return st;
    const int64_t t = c->t_warmup + 1;
    onebit::WarmupParams P;
    P.tiles = c->tiles();
    for (int w = 0; w < OB_MAX_WORKERS; ++w) P.g[w] = w < c->plan.W ? d_grads[w] : nullptr;
    P.m = c->m();
    P.v = c->v();
    P.p = c->params;
    P.W = c->plan.W;
    P.beta1 = c->beta1;
    P.beta2 = c->beta2;
    P.c1 = c->c1;
    P.c2 = c->c2;
    P.bc1 = (float)(1.0 - std::pow((double)c->beta1, (double)t));
    P.bc2 = (float)(1.0 - std::pow((double)c->beta2, (double)t));
    P.eps = c->eps;
    P.lr = c->lr;
    if (c->n_tiles() > 0 && !c->lamb) {
        KernelTimer k(c, OB_K_WARMUP);
        onebit::ob_warmup_kernel<<<grid1(c->n_tiles()), kThreads, 0, c->stream>>>(P);
        k.stop();
        if ((st = fail_cuda(c, cudaGetLastError())) != OB_OK) return st;
    }
    if (c->n_tiles() > 0 && c->lamb) {
        // 1-bit LAMB's warmup: the moments and each tensor's trust ratio,
        // then the step with the layerwise rates
        onebit::LambWarmupParams L{};
        L.w = P;
        L.partial = c->partial_lamb();
        L.n_tiles = c->n_tiles();
        L.sums = c->lamb_sums();
        L.T = c->plan.T;
        L.tensor_tile_begin = c->tensor_tile_begin();
        L.ratio = c->ratio();
        KernelTimer k(c, OB_K_WARMUP);
        onebit::ob_lamb_moments_kernel<<<grid1(c->n_tiles()), kThreads, 0, c->stream>>>(L);
        cudaError_t e = cudaGetLastError();
        if (e == cudaSuccess)  // ||p||^2 and ||r||^2 per tensor
            e = launch(onebit::ob_scale_kernel, range_sum_geometry(c->plan.T, 2, c->plan.tensor_max_seg),
                       tensor_sum_params(c, c->partial_lamb(), 2, c->lamb_sums()), c->stream);
        if (e == cudaSuccess) {
            onebit::ob_lamb_step_kernel<<<grid1(c->n_tiles()), kThreads, 0, c->stream>>>(L);
            e = cudaGetLastError();
        }
        k.stop();
        if ((st = fail_cuda(c, e)) != OB_OK) return st;
    }
    c->pnorm_valid = false;
    c->t_warmup = t;
    return OB_OK;
}

ob_status ob_freeze_variance(ob_ctx *c) {
    NvtxCall nvtx("ob_freeze_variance");
    ob_status st = check_ctx(c);
    if (st != OB_OK) return st;
    if (c->frozen || c->t_warmup < 1 || c->split_stage != 0) return OB_ERR_PHASE;
    DeviceGuard dg(c->device);
    if (!dg.ok) return fail_cuda(c, cudaErrorInvalidDevice);
    const float bc2 = (float)(1.0 - std::pow((double)c->beta2, (double)c->t_warmup));
    if (c->n_tiles() > 0) {
        KernelTimer k(c, OB_K_FREEZE);
        onebit::ob_freeze_kernel<<<grid1(c->n_tiles()), kThreads, 0, c->stream>>>(c->tiles(), c->v(),
                                                                               bc2, c->eps);
        k.stop();
        if ((st = fail_cuda(c, cudaGetLastError())) != OB_OK) return st;
    }
    // e_w = 0 and e_s = 0: zero the lazy values and their scales; clear the
    // last step's words and scales.
    const Carve &cv = c->cv;
    cudaError_t e = cudaMemsetAsync(c->x(), 0, cv.bits - cv.x, c->stream);  // x, y
    if (e == cudaSuccess) e = cudaMemsetAsync(c->bits(), 0, cv.partial_w - cv.bits, c->stream);
    if ((st = fail_cuda(c, e)) != OB_OK) return st;
    c->frozen = true;
    c->dnorm_valid = false;
    if (c->lamb && !c->lamb_frozen && (st = launch_lamb_norms(c, true, true)) != OB_OK) return st;
    return OB_OK;
}

ob_status ob_compressed_step(ob_ctx *c, const float *const *d_grads) {
    NvtxCall nvtx("ob_compressed_step");
    ob_status st = check_ctx(c);
    if (st != OB_OK) return st;
    if (!c->frozen || c->split_stage != 0) return OB_ERR_PHASE;
    if ((st = check_grads(c, d_grads)) != OB_OK) return st;
    DeviceGuard dg(c->device);
    if (!dg.ok) return fail_cuda(c, cudaErrorInvalidDevice);
    if ((st = ensure_lamb_norms(c)) != OB_OK) return st;
    // graph replay unless profiling, or unless the caller is capturing the
    // stream into a graph of its own (then the launches are captured)
    cudaStreamCaptureStatus capture = cudaStreamCaptureStatusNone;
    if (c->use_graph && !c->profiling &&
        (st = fail_cuda(c, cudaStreamIsCapturing(c->stream, &capture))) != OB_OK)
        return st;
    if (c->use_graph && !c->profiling && capture == cudaStreamCaptureStatusNone) {
        if ((st = graph_step(c, d_grads)) != OB_OK) return st;
    } else {
        KernelTimer pack(c, OB_K_PACK);
        if ((st = launch_pack(c, d_grads, 0, 0, c->n_tiles())) != OB_OK) return st;
        if ((st = launch_after_pack(c, pack)) != OB_OK) return st;
    }
    c->m_dense = false;
    c->t_compressed += 1;
    return OB_OK;
}

// ------------------------------------------------------- the split step
//
// One compressed step in two calls for a data-parallel run in which each
// process computes some of the workers (see onebit.h).  Host code only:
// the step's own kernels, the worker-stage ones launched on a view of the
// worker rows [w_begin, w_begin + w_count) as if those were all workers.

ob_status ob_worker_stage(ob_ctx *c, const float *const *d_grads, int w_begin, int w_count) {
    NvtxCall nvtx("ob_worker_stage");
    ob_status st = check_ctx(c);
    if (st != OB_OK) return st;
    if (!c->frozen || c->split_stage != 0) return OB_ERR_PHASE;
    const int W = c->plan.W;
    if (w_begin < 0 || w_count < 0 || w_begin > W - w_count || !d_grads) return OB_ERR_INVALID_ARG;
    if (c->plan.n_pad > 0)
        for (int w = w_begin; w < w_begin + w_count; ++w) {
            if (!d_grads[w]) return OB_ERR_INVALID_ARG;
            if (!aligned(d_grads[w], 16)) return OB_ERR_ALIGN;
        }
    DeviceGuard dg(c->device);
    if (!dg.ok) return fail_cuda(c, cudaErrorInvalidDevice);
    if ((st = ensure_lamb_norms(c)) != OB_OK) return st;
    const size_t n = (size_t)c->plan.n_pad, T = (size_t)c->plan.T, nt = (size_t)c->n_tiles();
    if (w_count > 0 && nt > 0) {
        // the step's worker-stage kernel on a view of the worker rows: the
        // rows [w_begin, w_begin + w_count) of x, bits, the scales, the
        // partial sums and the scales, as if they were all workers
        onebit::PackParams P = pack_params(c, d_grads, 0, 0);
        for (int i = 0; i < OB_MAX_WORKERS; ++i) P.g[i] = i < w_count ? d_grads[w_begin + i] : nullptr;
        P.x = c->x() + (size_t)w_begin * n;
        P.bits = c->bits() + (size_t)w_begin * (n / 32);
        P.s_prev = c->s_prev() + (size_t)w_begin * T;
        P.partial = c->partial_w() + (size_t)w_begin * nt;
        P.W = w_count;
        if (c->peer) {  // every chunk's words straight to the process serving it
            P.n_shards = c->n_shards;
            for (int q = 0; q < c->n_shards; ++q) {
                P.shard_end[q] = shard_tile_end(c->plan, c->n_shards, q);
                P.dest[q] = c->peer_bits[q] + (size_t)w_begin * (n / 32);
            }
        }
        KernelTimer k(c, OB_K_PACK);
        const cudaError_t e = launch(onebit::ob_pack_kernel, pack_geometry((int)nt), P, c->stream);
        k.stop();
        if ((st = fail_cuda(c, e)) != OB_OK) return st;
    }
    if (w_count > 0) {
        onebit::ScaleParams S = worker_scale_params(c);
        S.partial = c->partial_w() + (size_t)w_begin * nt;
        S.out_prev = c->s_prev() + (size_t)w_begin * T;
        S.out_last = c->s_last() + (size_t)w_begin * T;
        S.rows = w_count;
        KernelTimer k(c, OB_K_PACK_SCALE);
        const cudaError_t e = launch(onebit::ob_scale_kernel,
                                     range_sum_geometry((int)T, w_count, c->plan.tensor_max_seg), S,
                                     c->stream);
        k.stop();
        if ((st = fail_cuda(c, e)) != OB_OK) return st;
    }
    c->split_stage = 1;
    return OB_OK;
}

ob_status ob_worker_exchange_buffers(ob_ctx *c, uint32_t **d_bits, size_t *bits_row_bytes,
                                     float **d_scales, size_t *scales_row_bytes) {
    ob_status st = check_ctx(c);
    if (st != OB_OK) return st;
    if (!d_bits || !bits_row_bytes || !d_scales || !scales_row_bytes) return OB_ERR_INVALID_ARG;
    *d_bits = c->bits();
    *bits_row_bytes = (size_t)(c->plan.n_pad / 32) * 4;
    *d_scales = c->s_prev();
    *scales_row_bytes = (size_t)c->plan.T * 4;
    return OB_OK;
}

ob_status ob_set_server_shard(ob_ctx *c, int n_shards, int shard) {
    ob_status st = check_ctx(c);
    if (st != OB_OK) return st;
    if (n_shards < 1 || shard < 0 || shard >= n_shards) return OB_ERR_INVALID_ARG;
    if (c->split_stage != 0) return OB_ERR_PHASE;
    if (c->peer && n_shards != c->n_shards) return OB_ERR_PHASE;  // peers were set for the old split
    shard_chunks(c->plan, n_shards, shard, &c->chunk_lo, &c->chunk_hi);
    c->n_shards = n_shards;
    c->shard = shard;
    return OB_OK;
}

ob_status ob_set_peer_words(ob_ctx *c, int n_shards, uint32_t *const *d_worker_bits,
                            const uint32_t *const *d_server_bits) {
    ob_status st = check_ctx(c);
    if (st != OB_OK) return st;
    if (c->split_stage != 0) return OB_ERR_PHASE;
    if (n_shards == 0) {
        c->peer = false;
        return OB_OK;
    }
    if (n_shards != c->n_shards || n_shards > OB_MAX_WORKERS || !d_worker_bits || !d_server_bits)
        return OB_ERR_INVALID_ARG;
    for (int q = 0; q < n_shards; ++q) {
        if (!d_worker_bits[q] || !d_server_bits[q]) return OB_ERR_INVALID_ARG;
        if (!aligned(d_worker_bits[q], 16) || !aligned(d_server_bits[q], 16)) return OB_ERR_ALIGN;
    }
    try {
        host_alloc_point();
        c->peer_bits.assign(d_worker_bits, d_worker_bits + n_shards);
        c->peer_sbits.assign(d_server_bits, d_server_bits + n_shards);
    } catch (const std::bad_alloc &) {
        return OB_ERR_OOM;
    }
    c->peer = true;
    return OB_OK;
}

ob_status ob_server_shard_range(int n_tensors, const int64_t *numel, int W, int n_shards, int shard,
                                int *chunk_begin, int *chunk_end, int64_t *word_begin,
                                int64_t *word_end) {
    if (!chunk_begin || !chunk_end || !word_begin || !word_end) return OB_ERR_INVALID_ARG;
    if (n_shards < 1 || shard < 0 || shard >= n_shards) return OB_ERR_INVALID_ARG;
    try {
        Plan pl;
        ob_status st = make_plan(n_tensors, numel, W, true, &pl);
        if (st != OB_OK) return st;
        shard_chunks(pl, n_shards, shard, chunk_begin, chunk_end);
        *word_begin = chunk_first_word(pl, *chunk_begin);
        *word_end = chunk_first_word(pl, *chunk_end);
    } catch (const std::bad_alloc &) {
        return OB_ERR_OOM;
    }
    return OB_OK;
}

ob_status ob_server_stage(ob_ctx *c) {
    NvtxCall nvtx("ob_server_stage");
    ob_status st = check_ctx(c);
    if (st != OB_OK) return st;
    if (c->split_stage != 1) return OB_ERR_PHASE;
    DeviceGuard dg(c->device);
    if (!dg.ok) return fail_cuda(c, cudaErrorInvalidDevice);
    const Plan &pl = c->plan;
    const int C = pl.T * pl.W;
    const int lo = c->chunk_lo, hi = c->chunk_hi < 0 ? C : c->chunk_hi;
    // the exchange filled the other workers' rows of s_prev; S_WORKER reads
    // the copy in s_last
    cudaError_t e = cudaMemcpyAsync(c->s_last(), c->s_prev(), (size_t)pl.W * pl.T * 4,
                                    cudaMemcpyDeviceToDevice, c->stream);
    if ((st = fail_cuda(c, e)) != OB_OK) return st;
    // The server stage and its scales on the served chunks only: their
    // tiles are one contiguous range of the work list, launched from its
    // first tile (every index inside the kernels stays absolute), and their
    // scales one contiguous range of the chunk arrays.
    const int t_lo = pl.chunk_tile_begin[lo], t_hi = pl.chunk_tile_begin[hi];
    if (t_hi > t_lo) {
        onebit::ServerParams P = server_params(c);
        P.tile_base = t_lo;
        KernelTimer k(c, OB_K_SERVER);
        e = launch(onebit::ob_server_kernel, server_geometry(t_hi - t_lo, pl.W), P, c->stream);
        k.stop();
        if ((st = fail_cuda(c, e)) != OB_OK) return st;
    }
    if (hi > lo) {
        onebit::ScaleParams S = server_scale_params(c);
        S.range_begin = c->chunk_tile_begin() + lo;
        S.seg_base = c->chunk_seg_base() + lo;
        S.count = c->chunk_len() + lo;
        S.counter = c->counters_s() + lo;  // one row
        S.out_prev = c->sp_prev() + lo;
        S.out_last = c->sp_last() + lo;
        S.R = hi - lo;
        KernelTimer k(c, OB_K_SERVER_SCALE);
        e = launch(onebit::ob_scale_kernel, range_sum_geometry(hi - lo, 1, pl.chunk_max_seg), S, c->stream);
        k.stop();
        if ((st = fail_cuda(c, e)) != OB_OK) return st;
    }
    // The words and scales of the chunks served elsewhere are zero here, so
    // that summing every process's buffers gives every chunk its server's.
    const int64_t w_lo = chunk_first_word(pl, lo), w_hi = chunk_first_word(pl, hi);
    const int64_t words = pl.n_pad / 32;
    if (e == cudaSuccess && w_lo > 0) e = cudaMemsetAsync(c->sbits(), 0, (size_t)w_lo * 4, c->stream);
    if (e == cudaSuccess && w_hi < words)
        e = cudaMemsetAsync(c->sbits() + w_hi, 0, (size_t)(words - w_hi) * 4, c->stream);
    if (e == cudaSuccess && lo > 0) e = cudaMemsetAsync(c->sp_last(), 0, (size_t)lo * 4, c->stream);
    if (e == cudaSuccess && hi < C)
        e = cudaMemsetAsync(c->sp_last() + hi, 0, (size_t)(C - hi) * 4, c->stream);
    if ((st = fail_cuda(c, e)) != OB_OK) return st;
    c->split_stage = 2;
    return OB_OK;
}

ob_status ob_server_exchange_buffers(ob_ctx *c, uint32_t **d_sbits, size_t *sbits_bytes,
                                     float **d_scales, size_t *scales_bytes) {
    ob_status st = check_ctx(c);
    if (st != OB_OK) return st;
    if (!d_sbits || !sbits_bytes || !d_scales || !scales_bytes) return OB_ERR_INVALID_ARG;
    *d_sbits = c->sbits();
    *sbits_bytes = (size_t)(c->plan.n_pad / 32) * 4;
    *d_scales = c->sp_last();
    *scales_bytes = (size_t)c->plan.T * c->plan.W * 4;
    return OB_OK;
}

ob_status ob_apply_update(ob_ctx *c) {
    NvtxCall nvtx("ob_apply_update");
    ob_status st = check_ctx(c);
    if (st != OB_OK) return st;
    if (c->split_stage != 2) return OB_ERR_PHASE;
    DeviceGuard dg(c->device);
    if (!dg.ok) return fail_cuda(c, cudaErrorInvalidDevice);
    // the exchange completed the server scales in sp_last; the next server
    // stage decodes its y_prev with sp_prev
    cudaError_t e = cudaMemcpyAsync(c->sp_prev(), c->sp_last(), (size_t)c->plan.T * c->plan.W * 4,
                                    cudaMemcpyDeviceToDevice, c->stream);
    if ((st = fail_cuda(c, e)) != OB_OK) return st;
    if ((st = launch_apply(c)) != OB_OK) return st;
    c->split_stage = 0;
    c->m_dense = false;
    c->t_compressed += 1;
    return OB_OK;
}

ob_status ob_set_layerwise(ob_ctx *c, int mode) {
    ob_status st = check_ctx(c);
    if (st != OB_OK) return st;
    if (mode != OB_LAYERWISE_OFF && mode != OB_LAYERWISE_STEP && mode != OB_LAYERWISE_FROZEN)
        return OB_ERR_INVALID_ARG;
    if (c->t_warmup != 0 || c->t_compressed != 0 || c->frozen || c->split_stage != 0)
        return OB_ERR_PHASE;
    DeviceGuard dg(c->device);
    if (!dg.ok) return fail_cuda(c, cudaErrorInvalidDevice);
    try {
        host_alloc_point();
        const std::vector<float> ones((size_t)c->plan.T, 1.0f);  // empty tensors keep ratio 1
        cudaError_t e = cudaMemcpyAsync(c->ratio(), ones.data(), ones.size() * 4,
                                        cudaMemcpyHostToDevice, c->stream);
        if (e == cudaSuccess) e = cudaStreamSynchronize(c->stream);
        if ((st = fail_cuda(c, e)) != OB_OK) return st;
    } catch (const std::bad_alloc &) {
        return OB_ERR_OOM;
    }
    c->lamb = mode != OB_LAYERWISE_OFF;
    c->lamb_frozen = mode == OB_LAYERWISE_FROZEN;
    c->pnorm_valid = c->dnorm_valid = false;
    return OB_OK;
}

ob_status ob_graph_enable(ob_ctx *c, int on) {
    ob_status st = check_ctx(c);
    if (st != OB_OK) return st;
    c->use_graph = on != 0;
    return OB_OK;
}

ob_status ob_set_lr(ob_ctx *c, float lr) {
    ob_status st = check_ctx(c);
    if (st != OB_OK) return st;
    if (!std::isfinite(lr)) return OB_ERR_INVALID_ARG;
    c->lr = lr;
    return OB_OK;
}

ob_status ob_host_staging_bytes(const ob_ctx *c, size_t *bytes) {
    ob_status st = check_ctx(c);
    if (st != OB_OK) return st;
    if (!bytes) return OB_ERR_INVALID_ARG;
    *bytes = (size_t)2 * c->plan.W * kHostSlice * sizeof(float);
    return OB_OK;
}

ob_status ob_compressed_step_host(ob_ctx *c, const float *const *h_grads, void *d_staging,
                                  size_t staging_bytes, float *h_server_scales) {
    NvtxCall nvtx("ob_compressed_step_host");
    ob_status st = check_ctx(c);
    if (st != OB_OK) return st;
    if (!c->frozen || c->split_stage != 0) return OB_ERR_PHASE;
    if (!h_grads || !d_staging) return OB_ERR_INVALID_ARG;
    for (int w = 0; w < c->plan.W; ++w)
        if (!h_grads[w]) return OB_ERR_INVALID_ARG;
    if (!aligned(d_staging, kWsAlign)) return OB_ERR_ALIGN;
    const int W = c->plan.W;
    if (staging_bytes < (size_t)2 * W * kHostSlice * sizeof(float)) return OB_ERR_WORKSPACE;
    DeviceGuard dg(c->device);
    if (!dg.ok) return fail_cuda(c, cudaErrorInvalidDevice);
    if ((st = ensure_lamb_norms(c)) != OB_OK) return st;
    float *stage = static_cast<float *>(d_staging);
    // The copy stream must not overwrite staging still read by earlier work.
    cudaError_t e = cudaEventRecord(c->ev_start, c->stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(c->copy_stream, c->ev_start, 0);
    if ((st = fail_cuda(c, e)) != OB_OK) return st;
    KernelTimer pack(c, OB_K_PACK);
    const float *g[OB_MAX_WORKERS];
    for (size_t r = 0; r < c->host_runs.size(); ++r) {
        const Run &run = c->host_runs[r];
        const int slot = (int)(r & 1);
        if (r >= 2) e = cudaStreamWaitEvent(c->copy_stream, c->ev_consumed[slot], 0);
        const size_t bytes = (size_t)(run.elem_hi - run.elem_lo) * sizeof(float);
        for (int w = 0; w < W && e == cudaSuccess; ++w) {
            float *dst = stage + ((size_t)slot * W + w) * kHostSlice;
            e = cudaMemcpyAsync(dst, h_grads[w] + run.elem_lo, bytes, cudaMemcpyHostToDevice,
                                c->copy_stream);
            g[w] = dst;
        }
        if (e == cudaSuccess) e = cudaEventRecord(c->ev_copied[slot], c->copy_stream);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(c->stream, c->ev_copied[slot], 0);
        if ((st = fail_cuda(c, e)) != OB_OK) return st;
        if ((st = launch_pack(c, g, run.elem_lo, run.tile_lo, run.tile_hi)) != OB_OK) return st;
        if ((st = fail_cuda(c, cudaEventRecord(c->ev_consumed[slot], c->stream))) != OB_OK) return st;
    }
    if ((st = launch_after_pack(c, pack)) != OB_OK) return st;
    c->m_dense = false;
    c->t_compressed += 1;
    if (h_server_scales)
        e = cudaMemcpyAsync(h_server_scales, c->sp_last(),
                            (size_t)c->plan.T * W * sizeof(float), cudaMemcpyDeviceToHost, c->stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(c->stream);
    return fail_cuda(c, e);
}

ob_status ob_read_state(ob_ctx *c, int kind, int index, void *host_dst, size_t bytes) {
    ob_status st = check_ctx(c);
    if (st != OB_OK) return st;
    if (!host_dst) return OB_ERR_INVALID_ARG;
    const size_t want = state_bytes(c, kind);
    if (want == 0 || bytes != want) return OB_ERR_INVALID_ARG;
    const bool indexed = kind == OB_STATE_E_WORKER || kind == OB_STATE_BITS_WORKER;
    if (indexed ? (index < 0 || index >= c->plan.W) : index != 0) return OB_ERR_INVALID_ARG;
    if (kind == OB_STATE_V && c->frozen) return OB_ERR_PHASE;
    if (kind == OB_STATE_D && !c->frozen) return OB_ERR_PHASE;
    if (kind == OB_STATE_STEP) {
        const int64_t v[3] = {c->t_warmup, c->t_compressed, c->frozen ? 1 : 0};
        std::memcpy(host_dst, v, sizeof(v));
        return OB_OK;
    }
    DeviceGuard dg(c->device);
    if (!dg.ok) return fail_cuda(c, cudaErrorInvalidDevice);
    if ((st = fail_cuda(c, cudaStreamSynchronize(c->stream))) != OB_OK) return st;
    const size_t n = (size_t)c->plan.n_pad;
    try {
        if (kind == OB_STATE_E_WORKER)
            return read_error(c, c->x() + (size_t)index * n, c->s_prev() + (size_t)index * c->plan.T,
                              1, 0, static_cast<float *>(host_dst));
        if (kind == OB_STATE_E_SERVER)
            return read_error(c, c->y(), c->sp_prev(), c->plan.W, 1, static_cast<float *>(host_dst));
        if (kind == OB_STATE_M && !c->m_dense)
            return read_decoded(c, static_cast<float *>(host_dst),
                                [&](const Run &r, float *out, int64_t base) {
                                    launch_decode_momentum(c, r.tile_lo, r.tile_hi, out, base);
                                });
    } catch (const std::bad_alloc &) {
        return OB_ERR_OOM;
    }
    const void *src = nullptr;
    switch (kind) {
    case OB_STATE_P: src = c->params; break;
    case OB_STATE_M: src = c->m(); break;
    case OB_STATE_V: case OB_STATE_D: src = c->v(); break;
    case OB_STATE_S_WORKER: src = c->s_last(); break;
    case OB_STATE_S_SERVER: src = c->sp_last(); break;
    case OB_STATE_BITS_WORKER: src = c->bits() + (size_t)index * (n / 32); break;
    case OB_STATE_BITS_SERVER: src = c->sbits(); break;
    case OB_STATE_RATIO: src = c->ratio(); break;
    default: return OB_ERR_INVALID_ARG;
    }
    cudaError_t e = cudaMemcpyAsync(host_dst, src, bytes, cudaMemcpyDeviceToHost, c->stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(c->stream);
    return fail_cuda(c, e);
}

ob_status ob_write_state(ob_ctx *c, int kind, int index, const void *host_src, size_t bytes) {
    ob_status st = check_ctx(c);
    if (st != OB_OK) return st;
    if (c->split_stage != 0) return OB_ERR_PHASE;
    if (!host_src) return OB_ERR_INVALID_ARG;
    const size_t want = state_bytes(c, kind);
    if (want == 0 || bytes != want) return OB_ERR_INVALID_ARG;
    const bool indexed = kind == OB_STATE_E_WORKER;
    if (indexed ? (index < 0 || index >= c->plan.W) : index != 0) return OB_ERR_INVALID_ARG;
    if (kind == OB_STATE_V && c->frozen) return OB_ERR_PHASE;
    if (kind == OB_STATE_D && !c->frozen) return OB_ERR_PHASE;
    if (kind == OB_STATE_STEP) {
        int64_t v[3];
        std::memcpy(v, host_src, sizeof(v));
        if (v[0] < 0 || v[1] < 0 || (v[2] != 0 && v[2] != 1) || (v[2] == 1 && v[0] < 1) ||
            (v[2] == 0 && v[1] != 0))
            return OB_ERR_INVALID_ARG;
        c->t_warmup = v[0];
        c->t_compressed = v[1];
        c->frozen = v[2] == 1;
        return OB_OK;
    }
    DeviceGuard dg(c->device);
    if (!dg.ok) return fail_cuda(c, cudaErrorInvalidDevice);
    const size_t n = (size_t)c->plan.n_pad;
    void *dst = nullptr;
    cudaError_t e = cudaSuccess;
    switch (kind) {
    case OB_STATE_P: dst = c->params; c->pnorm_valid = false; break;
    case OB_STATE_M: dst = c->m(); c->m_dense = true; break;
    case OB_STATE_V: dst = c->v(); break;
    case OB_STATE_D: dst = c->v(); c->dnorm_valid = false; break;
    case OB_STATE_E_WORKER:
        // stored as (x, s) with s = 0, which decodes to x exactly
        dst = c->x() + (size_t)index * n;
        e = cudaMemsetAsync(c->s_prev() + (size_t)index * c->plan.T, 0, (size_t)c->plan.T * 4,
                            c->stream);
        break;
    case OB_STATE_E_SERVER:
        dst = c->y();
        e = cudaMemsetAsync(c->sp_prev(), 0, (size_t)c->plan.T * c->plan.W * 4, c->stream);
        break;
    case OB_STATE_RATIO:  // state only when the ratios are kept at the freeze
        if (!c->lamb_frozen) return OB_ERR_INVALID_ARG;
        dst = c->ratio();
        break;
    default:
        return OB_ERR_INVALID_ARG;
    }
    if (e == cudaSuccess) e = cudaMemcpyAsync(dst, host_src, bytes, cudaMemcpyHostToDevice, c->stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(c->stream);
    return fail_cuda(c, e);
}

ob_status ob_profile_enable(ob_ctx *c, int on) {
    ob_status st = check_ctx(c);
    if (st != OB_OK) return st;
    c->profiling = on != 0;
    return OB_OK;
}

ob_status ob_profile_read(ob_ctx *c, double *ms, int64_t *launches, int reset) {
    ob_status st = check_ctx(c);
    if (st != OB_OK) return st;
    DeviceGuard dg(c->device);
    if (!dg.ok) return fail_cuda(c, cudaErrorInvalidDevice);
    if ((st = fail_cuda(c, cudaStreamSynchronize(c->stream))) != OB_OK) return st;
    for (auto &p : c->pending) {
        float t = 0.f;
        cudaError_t e = cudaEventElapsedTime(&t, p.second.first, p.second.second);
        if (e != cudaSuccess) return fail_cuda(c, e);
        c->kernel_ms[p.first] += t;
        c->kernel_launches[p.first] += 1;
        c->event_pool.push_back(p.second.first);
        c->event_pool.push_back(p.second.second);
    }
    c->pending.clear();
    for (int k = 0; k < OB_NUM_KERNELS; ++k) {
        if (ms) ms[k] = c->kernel_ms[k];
        if (launches) launches[k] = c->kernel_launches[k];
        if (reset) {
            c->kernel_ms[k] = 0;
            c->kernel_launches[k] = 0;
        }
    }
    return OB_OK;
}

}  // extern "C"

// ============================================ compressor without allocation
//
// Scratch for ob_onebit_compress_static: one fp64 partial sum per 4096-element
// tile, in a file-scope device array (OB_STATIC_MAX_ELEMENTS / 4096 entries,
// 128 KiB).  It lives in the library's module, so every GPU that loads the
// library holds it until the process exits.  Host code may not pass the
// array's name to a kernel (on the host it is only a stand-in); its device
// address is looked up with cudaGetSymbolAddress, with the device current,
// on every call: the lookup allocates nothing, and an address kept from an
// earlier call would be stale after the caller reset the device (the
// module is then loaded again, possibly elsewhere).

namespace {

constexpr int kStaticTiles = (int)(OB_STATIC_MAX_ELEMENTS / kTile);
static_assert((int64_t)kStaticTiles * kTile == OB_STATIC_MAX_ELEMENTS, "static scratch size");

}  // namespace

static __device__ __align__(256) double g_static_partial[kStaticTiles];

extern "C" ob_status ob_onebit_compress_static(const float *d_x, int64_t n, uint32_t *d_bits,
                                               float *d_error, float *d_scale, void *cuda_stream) {
    if (n < 0 || !d_scale) return OB_ERR_INVALID_ARG;
    if (n > OB_STATIC_MAX_ELEMENTS) return OB_ERR_WORKSPACE;  // larger than the built-in scratch
    if (n > 0 && (!d_x || !d_bits || !d_error)) return OB_ERR_INVALID_ARG;
    if (!aligned(d_x, 16) || !aligned(d_error, 16) || !aligned(d_bits, 4) || !aligned(d_scale, 4))
        return OB_ERR_ALIGN;
    void *addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_static_partial) != cudaSuccess || !addr) return OB_ERR_CUDA;
    double *scratch = static_cast<double *>(addr);
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    const int tiles = (int)((n + kTile - 1) / kTile);
    // Each launch's own status (cudaLaunchKernel returns it), so an error
    // left by unrelated earlier work is neither reported nor cleared here.
    if (tiles > 0) {
        void *args[] = {(void *)&d_x, (void *)&n, (void *)&d_bits, (void *)&scratch};
        if (cudaLaunchKernel((const void *)onebit::ob_compress_partial_kernel, dim3(tiles),
                             dim3(kThreads), args, 0, stream) != cudaSuccess)
            return OB_ERR_CUDA;
    }
    {
        int tiles_arg = tiles;
        void *args[] = {(void *)&scratch, (void *)&tiles_arg, (void *)&n, (void *)&d_scale};
        if (cudaLaunchKernel((const void *)onebit::ob_compress_scale_kernel, dim3(1),
                             dim3(kScaleThreads), args, 0, stream) != cudaSuccess)
            return OB_ERR_CUDA;
    }
    if (tiles > 0) {
        const float *scale_in = d_scale;
        void *args[] = {(void *)&d_x, (void *)&n, (void *)&scale_in, (void *)&d_error};
        if (cudaLaunchKernel((const void *)onebit::ob_compress_error_kernel, dim3(tiles),
                             dim3(kThreads), args, 0, stream) != cudaSuccess)
            return OB_ERR_CUDA;
    }
    return OB_OK;
}
