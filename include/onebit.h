/*
 * onebit.h -- C ABI of libonebit: the compression-phase step of 1-bit Adam
 * on one NVIDIA B200 (sm_100a), with W data-parallel workers simulated as W
 * state buffers in the GPU's HBM.
 *
 * The method is the one on the review page "1-bit Adam: Communication
 * Efficient Large-Scale Training with Adam's Convergence Speed" ([1BA]):
 *   - [1BA, Proposed method, 1]: training runs full-precision Adam for a
 *     warmup (typically 20% of the steps), then 1-bit compressed momentum
 *     SGD for the rest;
 *   - [1BA, Abstract; Proposed method, 2]: Adam's variance is stable after
 *     the warmup and is frozen, becoming the fixed preconditioner;
 *   - [1BA, Proposed method, 3]: error-compensated 1-bit compression is
 *     applied to the momentum;
 *   - [1BA, Proposed method, 4]: a custom compressed collective (a worker
 *     stage and a server stage) averages the compressed momentum.
 * The calls below follow that two-phase statement:
 *   ob_create -> ob_warmup_adam_step* -> ob_freeze_variance ->
 *   ob_compressed_step* (state machine enforced; OB_ERR_PHASE otherwise),
 * where a compressed step may also be taken as the split step
 * (ob_worker_stage, ob_server_stage, ob_apply_update, with the caller's
 * exchanges between them) when the workers are spread over processes.
 *
 * Conventions shared by every call
 *   - Every call returns an ob_status and never aborts, throws or exits.
 *   - A "tensor list" is n_tensors >= 1 tensors of numel[t] >= 0 fp32
 *     elements.  Each tensor is an independent problem: its own worker
 *     scales, sign packing and server chunks.
 *   - Padded layout: all flat per-parameter buffers (parameters, gradients,
 *     dense state) hold the tensors back to back, tensor t starting at
 *     element offset[t] (a multiple of OB_TENSOR_ALIGN), its numel[t]
 *     elements followed by padding up to the next multiple of
 *     OB_TENSOR_ALIGN.  n_padded is the total.  Padding entries are never
 *     read into any result and never updated.  ob_layout gives offsets.
 *   - Packed sign words (uint32): bit k of word i of tensor t is element
 *     32*i + k of that tensor; tensor t's words start at word offset[t]/32;
 *     bit 1 means +1 (x >= 0, so sign(0) = +1), bit 0 means -1; padding
 *     bits are 0.
 *   - Device pointers must be 16-byte aligned (OB_ERR_ALIGN otherwise); the
 *     workspace 256-byte aligned.  libonebit never allocates or frees device
 *     memory: the caller owns parameters, gradients and workspace.
 *   - All GPU work is queued on the CUDA stream given to ob_create; the
 *     step calls return once it is queued.  Launch errors are returned at
 *     once; faults of queued work surface as OB_ERR_CUDA from the next call
 *     that synchronizes (ob_read_state / ob_write_state /
 *     ob_compressed_step_host / ob_profile_read).  After OB_ERR_CUDA a
 *     context only accepts ob_destroy.
 *   - A context is not thread-safe; use it from one host thread at a time.
 *     Calls on a destroyed or unknown context return OB_ERR_INVALID_ARG.
 */
#ifndef ONEBIT_H
#define ONEBIT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define OB_API __attribute__((visibility("default")))
#else
#define OB_API
#endif

#define OB_ABI_VERSION 1
#define OB_MAX_WORKERS 64     /* W is 1..OB_MAX_WORKERS */
#define OB_TENSOR_ALIGN 128   /* elements; tensor offsets are multiples of this */

typedef struct ob_ctx ob_ctx; /* opaque */

typedef enum ob_status {
    OB_OK = 0,
    OB_ERR_INVALID_ARG = 1,    /* bad count, size, index, kind or NULL pointer; unknown context */
    OB_ERR_PHASE = 2,          /* call out of the warmup -> freeze -> compressed order */
    OB_ERR_ALIGN = 3,          /* a device pointer is not 16-byte (workspace: 256-byte) aligned */
    OB_ERR_WORKSPACE = 4,      /* workspace or staging buffer smaller than required */
    OB_ERR_OOM = 5,            /* host memory allocation failed */
    OB_ERR_CUDA = 6,           /* a CUDA call failed; the context is now unusable */
    OB_ERR_DEVICE_TIMEOUT = 7  /* reserved: no kernel of this library waits on anything */
} ob_status;

/* Kinds of state for ob_read_state / ob_write_state. */
typedef enum ob_state_kind {
    OB_STATE_P = 0,           /* parameters p, float[n_padded] (the caller's buffer)           rw */
    OB_STATE_M = 1,           /* momentum m, float[n_padded]                                    rw */
    OB_STATE_V = 2,           /* Adam variance v, float[n_padded]; before the freeze only       rw */
    OB_STATE_D = 3,           /* frozen denominator d = sqrt(v/bc2)+eps; after the freeze only  rw */
    OB_STATE_E_WORKER = 4,    /* index w: worker w's error feedback e_w, float[n_padded]        rw */
    OB_STATE_E_SERVER = 5,    /* server error feedback e_s, float[n_padded]                     rw */
    OB_STATE_S_WORKER = 6,    /* last step's worker scales, float[W][n_tensors]                 r  */
    OB_STATE_S_SERVER = 7,    /* last step's server chunk scales, float[n_tensors][W]           r  */
    OB_STATE_BITS_WORKER = 8, /* index w: last step's packed worker signs, uint32[n_padded/32]  r  */
    OB_STATE_BITS_SERVER = 9, /* last step's packed server signs, uint32[n_padded/32]           r  */
    OB_STATE_STEP = 10,       /* int64[3]: {warmup steps taken, compressed steps taken, frozen} rw */
    OB_STATE_RATIO = 11       /* last step's 1-bit LAMB trust ratios, float[n_tensors] (1 while
                                 layerwise rates are off, before the first step, for empty
                                 tensors); written only in OB_LAYERWISE_FROZEN, where they
                                 are state (the ratios kept at the freeze)                     r  */
} ob_state_kind;

/* Kernels timed by the profiling counters (ob_profile_read). */
typedef enum ob_kernel_id {
    OB_K_WARMUP = 0,          /* ob_warmup_adam_step */
    OB_K_FREEZE = 1,          /* ob_freeze_variance */
    OB_K_PACK = 2,            /* worker stage: momentum, error, signs, partial sums of squares */
    OB_K_PACK_SCALE = 3,      /* worker scales from the partial sums (ob_scale_kernel) */
    OB_K_SERVER = 4,          /* server stage: average, server error, signs, partial sums */
    OB_K_SERVER_SCALE = 5,    /* server chunk scales from the partial sums (ob_scale_kernel) */
    OB_K_APPLY = 6,           /* gather, decode and preconditioned update (1-bit LAMB: with its
                                 norm sums) */
    OB_NUM_KERNELS = 7
} ob_kernel_id;

/* Name of a status code (static string; never NULL). */
OB_API const char *ob_status_string(ob_status status);

/* OB_ABI_VERSION of the loaded library. */
OB_API int ob_abi_version(void);

/* Padded layout of a tensor list (host only, no GPU needed).
 * numel: n_tensors counts (>= 0).  tensor_offsets (out, may be NULL):
 * n_tensors element offsets.  n_padded (out): total padded elements.
 * OB_ERR_INVALID_ARG for n_tensors < 1, a negative count, NULL numel or
 * n_padded, or a total above 2^40 elements. */
OB_API ob_status ob_layout(int n_tensors, const int64_t *numel, int64_t *tensor_offsets,
                    int64_t *n_padded);

/* Server j's chunk of a tensor of numel elements split among W servers
 * (host only).  [1BA, Proposed method, 4]: with nw = ceil(numel/32) sign
 * words, each server owns cw = roundup(ceil(nw/W), 4) words; server j owns
 * elements [min(numel, 32*j*cw), min(numel, 32*(j+1)*cw)).  Chunks start on
 * 128-element boundaries, so no sign word or 16-byte word group is split;
 * trailing servers may own nothing.  OB_ERR_INVALID_ARG for numel < 0, W
 * outside 1..OB_MAX_WORKERS, j outside 0..W-1 or NULL outputs. */
OB_API ob_status ob_chunk_range(int64_t numel, int W, int j, int64_t *begin, int64_t *end);

/* Bytes of device workspace ob_create needs for this tensor list and W
 * (host only).  The workspace holds every piece of optimizer state except
 * the parameters: m, v/d, the W worker error buffers, the server error,
 * packed signs, scales, per-tile partial sums and the tile work list. */
OB_API ob_status ob_workspace_bytes(int n_tensors, const int64_t *numel, int W, size_t *bytes);

/* Create a context.  numel: as for ob_layout (copied).  W: simulated
 * workers, 1..OB_MAX_WORKERS.  beta1, beta2 in [0, 1), eps > 0, lr: Adam
 * hyperparameters (the same lr drives the compressed phase).  d_params:
 * device float[n_padded] in the padded layout, caller-owned, updated in
 * place by the step calls (NULL allowed only when n_padded is 0).  d_workspace: device buffer of workspace_bytes
 * >= ob_workspace_bytes(...), 256-byte aligned, caller-owned, not touched
 * by the caller while the context lives.  cuda_stream: cudaStream_t (NULL =
 * legacy default stream) on the current device; every call of this
 * context queues its work there.  The call uploads the work list and
 * zeroes the state, then waits for the stream.  *out receives the context.
 * Errors: OB_ERR_INVALID_ARG, OB_ERR_ALIGN, OB_ERR_WORKSPACE, OB_ERR_OOM,
 * OB_ERR_CUDA. */
OB_API ob_status ob_create(int n_tensors, const int64_t *numel, int W, float beta1, float beta2,
                    float eps, float lr, float *d_params, void *d_workspace,
                    size_t workspace_bytes, void *cuda_stream, ob_ctx **out);

/* Destroy a context (NULL and unknown pointers are ignored).  Waits for the
 * context's stream; frees only host-side objects. */
OB_API void ob_destroy(ob_ctx *ctx);

/* One full-precision Adam step on the averaged gradient
 * [1BA, Proposed method, 1].  d_grads: host array of W device pointers,
 * each a float[n_padded] gradient in the padded layout (read only).  With
 * t the new step count, bc1 = 1 - beta1^t, bc2 = 1 - beta2^t:
 *   gbar = (g_0 + ... + g_{W-1}) / W,  m = beta1 m + (1-beta1) gbar,
 *   v = beta2 v + (1-beta2) gbar^2,    p -= lr (m/bc1) / (sqrt(v/bc2) + eps).
 * Pointers may be NULL when n_padded is 0.  OB_ERR_PHASE after the freeze. */
OB_API ob_status ob_warmup_adam_step(ob_ctx *ctx, const float *const *d_grads);

/* Freeze the variance [1BA, Abstract; Proposed method, 2]: d = sqrt(v /
 * bc2(Tw)) + eps replaces v (Tw = warmup steps taken), every worker and
 * server error is set to 0, and m is kept.  OB_ERR_PHASE if no warmup step
 * was taken or the variance is already frozen. */
OB_API ob_status ob_freeze_variance(ob_ctx *ctx);

/* One compression-phase step [1BA, Proposed method, 1-4], all on the GPU:
 *   worker stage, per worker w and tensor t:
 *     m_w = beta1 m + (1-beta1) g_w;  x = m_w + e_w;
 *     s_w = ||x||_2 / sqrt(numel_t);  signs of x packed 32 per word;
 *     e_w = x - sign(x) s_w;
 *   server stage, per tensor t and server chunk j:
 *     y = (sum over w in order of sign_w s_w) / W + e_s;
 *     s'_j = ||y over chunk j||_2 / sqrt(len_j) (0 for an empty chunk);
 *     signs of y packed;  e_s = y - sign(y) s'_j;
 *   gather and update:  m_hat = sign(y) s'_j;  p -= lr (m_hat / d);
 *     m = m_hat for every worker.
 * d_grads: as for ob_warmup_adam_step.  OB_ERR_PHASE before the freeze. */
OB_API ob_status ob_compressed_step(ob_ctx *ctx, const float *const *d_grads);

/* Bytes of device staging ob_compressed_step_host needs (host only). */
OB_API ob_status ob_host_staging_bytes(const ob_ctx *ctx, size_t *bytes);

/* The compression-phase step with the gradients in HOST memory.  h_grads:
 * host array of W host pointers, each float[n_padded] in the padded layout
 * (page-locked memory lets the copies overlap the worker stage).  The
 * gradients are copied to the GPU in slices through d_staging (device,
 * caller-owned, >= ob_host_staging_bytes, 256-byte aligned) on a second
 * stream, overlapping the worker stage of earlier slices; the rest of the
 * step is ob_compressed_step's.  h_server_scales (may be NULL) receives the
 * step's server chunk scales, float[n_tensors][W].  The call returns when
 * the step is complete on the GPU.  Errors as ob_compressed_step, plus
 * OB_ERR_WORKSPACE for a small staging buffer. */
OB_API ob_status ob_compressed_step_host(ob_ctx *ctx, const float *const *h_grads, void *d_staging,
                                  size_t staging_bytes, float *h_server_scales);

/* --------------------------------------------------------------------
 * The split step: one compressed step in three calls, for a data-parallel
 * run over G processes (one per GPU) in which process r computes the
 * workers [w_begin, w_begin + w_count) and serves one contiguous range of
 * the server chunks -- the worker stage and the server stage of the
 * compressed collective [1BA, Proposed method, 4], with the caller moving
 * each stage's outputs between the processes:
 *
 *   ob_set_server_shard(ctx, G, r)                        once
 *   per step:
 *     ob_worker_stage(ctx, d_grads, w_begin, w_count)
 *     all-gather of the worker rows (ob_worker_exchange_buffers)
 *     ob_server_stage(ctx)
 *     sum-all-reduce of ob_server_exchange_buffers (words as 32-bit
 *       integers, scales as floats)
 *     ob_apply_update(ctx)
 *
 * Every process holds a context over the whole tensor list with all W
 * workers' rows; p, m and d stay the same on every process.  Each server
 * word and scale is written by one process and is zero on the others, so
 * the sums are exact and the result equals ob_compressed_step over all W
 * workers bit for bit.  With G = 1 the server exchange is not needed.
 * While a split step is open (from ob_worker_stage to ob_apply_update)
 * only its next call, the exchange-buffer calls, ob_read_state and
 * ob_destroy are accepted; the other step calls, ob_set_server_shard and
 * ob_write_state return OB_ERR_PHASE.  Warmup steps need the gradients of
 * all W workers on every process (the warmup averages them in worker
 * order).  The server error (E_SERVER) of a process is this step's only on
 * the chunks it serves. */

/* Chunks [*chunk_begin, *chunk_end) of shard `shard` of n_shards, in flat
 * index t * W + j (tensor t, server j), and the server words
 * [*word_begin, *word_end) they cover.  The shards are contiguous in
 * (tensor, chunk) order, cut so that each holds about the same number of
 * 4096-element tiles; together they cover every chunk and word once.
 * Host only. */
OB_API ob_status ob_server_shard_range(int n_tensors, const int64_t *numel, int W, int n_shards,
                                       int shard, int *chunk_begin, int *chunk_end,
                                       int64_t *word_begin, int64_t *word_end);

/* Serve the chunks of shard `shard` of n_shards (ob_server_shard_range) in
 * the split step.  Default: every chunk.  OB_ERR_PHASE while a split step
 * is open. */
OB_API ob_status ob_set_server_shard(ob_ctx *ctx, int n_shards, int shard);

/* Worker stage of workers [w_begin, w_begin + w_count) (w_count may be 0):
 * momentum, error feedback, 1-bit compression and worker scales, as in
 * ob_compressed_step.  d_grads: host array of W device pointers, only the
 * entries of the range read (the others may be NULL).  For a list of more
 * than one tensor the momentum is first decoded into its dense buffer (one
 * extra pass of 4 bytes per parameter).  OB_ERR_PHASE before the freeze or
 * while a split step is open; OB_ERR_INVALID_ARG for a range outside
 * [0, W) or a NULL gradient in it. */
OB_API ob_status ob_worker_stage(ob_ctx *ctx, const float *const *d_grads, int w_begin, int w_count);

/* Device buffers of the worker stage's outputs, one row per worker, rows
 * adjacent (row w at base + w * row_bytes): *d_bits uint32[W][n_padded/32]
 * sign words, *d_scales float[W][n_tensors] worker scales.  Owned by the
 * context (inside its workspace); valid until ob_destroy. */
OB_API ob_status ob_worker_exchange_buffers(ob_ctx *ctx, uint32_t **d_bits, size_t *bits_row_bytes,
                                            float **d_scales, size_t *scales_row_bytes);

/* Server stage of the served chunks, once every worker row holds this
 * step's words and scales: average, server error, re-compression and
 * server scales, as in ob_compressed_step; the words and scales of the
 * other chunks are set to 0.  OB_ERR_PHASE unless ob_worker_stage came
 * before. */
OB_API ob_status ob_server_stage(ob_ctx *ctx);

/* Device buffers of the server stage's outputs: *d_sbits uint32[n_padded/32]
 * server sign words, *d_scales float[n_tensors][W] server scales.  Owned
 * by the context; valid until ob_destroy. */
OB_API ob_status ob_server_exchange_buffers(ob_ctx *ctx, uint32_t **d_sbits, size_t *sbits_bytes,
                                            float **d_scales, size_t *scales_bytes);

/* Gather and update with every chunk's words and scales present; closes
 * the split step (the compressed step count advances).  OB_ERR_PHASE
 * unless ob_server_stage came before. */
OB_API ob_status ob_apply_update(ob_ctx *ctx);

/* The split step with the word exchanges fused into the kernels: the
 * worker stage's sign words of each chunk are stored straight into the
 * worker rows of the process serving it, and the update reads each chunk's
 * server words from the process serving it (copying them into this
 * context's server words, which the next step's momentum decode reads)
 * -- [1BA, Proposed method, 4]'s worker stage and gather, with the pack
 * and the unpack doing the transfers.  d_worker_bits[q] / d_server_bits[q]:
 * the buffers ob_worker_exchange_buffers / ob_server_exchange_buffers
 * return in the context serving shard q, as device addresses this process
 * can store to and load from (the same device, or another GPU's memory
 * mapped here, e.g. through CUDA IPC, reached with plain loads and
 * stores); the entry of this context's own shard may be its own buffers.
 * n_shards must be the shard count given to ob_set_server_shard (0 turns
 * this off).  With
 * it on, the caller exchanges only the worker scales (all-gather) and the
 * server scales (every process's chunk range to every process), each after
 * the stage that produced them: those exchanges also order the stages
 * across processes (a process's server stage must start after every
 * process's worker stage has finished storing into it, and the servers'
 * words must be complete before any update reads them).  A context's
 * worker rows then hold, for every worker including its own, only the
 * words of the chunks it serves.  OB_ERR_PHASE while
 * a split step is open; OB_ERR_INVALID_ARG for a shard count that differs
 * from the context's or a NULL buffer; OB_ERR_ALIGN for a buffer that is
 * not 16-byte aligned.  The library cannot check that the addresses point
 * at the right buffers. */
OB_API ob_status ob_set_peer_words(ob_ctx *ctx, int n_shards, uint32_t *const *d_worker_bits,
                                   const uint32_t *const *d_server_bits);

/* Copy one piece of state to host memory.  kind: ob_state_kind.  index:
 * the worker for OB_STATE_E_WORKER / OB_STATE_BITS_WORKER, else 0.  bytes:
 * must equal the size listed with the kind.  Waits for the stream first.
 * Error buffers are decoded on the GPU (padding entries read as 0).
 * OB_ERR_PHASE for V after / D before the freeze. */
OB_API ob_status ob_read_state(ob_ctx *ctx, int kind, int index, void *host_dst, size_t bytes);

/* Overwrite one piece of state from host memory (resume from a checkpoint,
 * or re-sync with another implementation).  Same arguments as
 * ob_read_state; the kinds marked r above are read only
 * (OB_ERR_INVALID_ARG).  OB_STATE_STEP takes {t_warmup >= 0,
 * t_compressed >= 0, frozen in {0,1}} with frozen requiring t_warmup >= 1.
 * Waits for the copy to finish. */
OB_API ob_status ob_write_state(ob_ctx *ctx, int kind, int index, const void *host_src, size_t bytes);

/* 1-bit LAMB: layerwise adaptive learning rates.  The 1-bit LAMB review
 * page ("1-bit LAMB: Communication Efficient Large-Scale Large-Batch
 * Training with LAMB's Convergence Speed", Abstract) keeps LAMB's
 * layerwise rates while the momentum is exchanged compressed; it prints no
 * update rule.  The rate taken is LAMB's trust ratio per tensor,
 *   ratio_t = ||p_t|| / ||u_t||   (1 when either norm is 0),
 * scaling that tensor's step: p -= (lr ratio_t) u.  In the warmup u is
 * Adam's direction m_hat / (sqrt(v_hat) + eps), the ratio recomputed every
 * step.  In the compression phase, mode
 *   OB_LAYERWISE_STEP    recomputes it every step with u = m_hat / d, m_hat
 *                        the momentum decoded from the compressed exchange
 *                        (the same on every worker), d the frozen
 *                        denominator;
 *   OB_LAYERWISE_FROZEN  keeps the last warmup step's ratios from the
 *                        freeze on, as the variance is kept (they are then
 *                        state: OB_STATE_RATIO can be written, for resume);
 *   OB_LAYERWISE_OFF     (the default) is 1-bit Adam.
 * Everything else (the compressed exchange, the errors, the freeze) is
 * 1-bit Adam's.  The trust ratios are read as OB_STATE_RATIO.  Only before
 * the first step: OB_ERR_PHASE afterwards; another mode OB_ERR_INVALID_ARG.
 * The ratios are rounded from fp64 sums of squares taken in an order of
 * the GPU's own, so they can differ from a sequential evaluation in the
 * last place. */
#define OB_LAYERWISE_OFF 0
#define OB_LAYERWISE_STEP 1
#define OB_LAYERWISE_FROZEN 2
OB_API ob_status ob_set_layerwise(ob_ctx *ctx, int mode);

/* Set the learning rate used by the following warmup and compressed steps
 * (learning-rate schedules).  OB_ERR_INVALID_ARG for a non-finite lr. */
OB_API ob_status ob_set_lr(ob_ctx *ctx, float lr);

/* Graph mode on (the default) or off.  While on, profiling is off and the
 * context's stream is not being captured by the caller, ob_compressed_step
 * replays the step's kernels as one CUDA graph, built at the first such
 * call: one launch instead of five, which matters for small tensor lists
 * where each kernel runs a few microseconds.  Changed gradient pointers,
 * the dense/lazy state of m and the learning rate are written into the
 * graph before each replay; the results are those of the ordinary
 * launches.  While the caller captures the stream (or with graph mode or
 * profiling off) the kernels are launched one by one, so they become part
 * of the caller's capture; a captured step keeps the launch parameters of
 * the step it was captured from (gradient pointers, learning rate, and
 * whether m is read densely, as only the first step after the warmup or a
 * write of M does), so capture a step after the first compressed one.
 * ob_compressed_step_host and the split step never use the graph. */
OB_API ob_status ob_graph_enable(ob_ctx *ctx, int on);

/* Turn per-kernel timing on or off.  While on, every step records CUDA
 * events between its kernels on the context's stream. */
OB_API ob_status ob_profile_enable(ob_ctx *ctx, int on);

/* Wait for the stream and return, per ob_kernel_id, the summed event time
 * in milliseconds (ms, may be NULL) and the number of launches (launches,
 * may be NULL) since profiling was enabled or last reset; reset != 0 clears
 * the counters afterwards.  Arrays have OB_NUM_KERNELS entries. */
OB_API ob_status ob_profile_read(ob_ctx *ctx, double *ms, int64_t *launches, int reset);

/* Name of a kernel id, or NULL for an unknown id. */
OB_API const char *ob_kernel_name(int kernel_id);

/* Test hook: make the countdown-th host allocation from now on fail with
 * OB_ERR_OOM (countdown <= 0 disarms).  Host memory only. */
OB_API void ob_test_fail_host_alloc(int countdown);

/* --------------------------------------------------------------------
 * A compressor that allocates nothing.
 *
 * Some callers cannot allocate device memory: a plugin inside a host
 * framework whose caching allocator has already reserved the GPU's memory
 * (a direct cudaMalloc there fails or fragments the pool), or a
 * latency-critical loop that cannot afford cudaMalloc's implicit device
 * synchronization.  For them this entry point needs no workspace at all:
 * the caller passes only inputs and outputs, and the scratch (one fp64
 * partial sum per 4096 elements) is a static device array of the library,
 * sized for OB_STATIC_MAX_ELEMENTS elements (128 KiB), which every GPU
 * that loads the library holds until the process exits.  The paper has no
 * counterpart to this call; it is the worker stage's compressor of
 * ob_compressed_step applied to a given x:
 *   s = ||x||_2 / sqrt(n);  bits: 1 where x >= 0;  e = x - sign(x) s.
 * The sign words are those of x bit for bit.  The fp64 sum of squares is
 * taken in an order of its own (per thread, then per tile, then over the
 * tiles in order), so s can differ from the workspace path's scale in the
 * last place (within 1e-6 relative); e is that path's bit for bit whenever
 * the two scales are equal.
 * d_x: device float[n] (16-byte aligned, no padding needed).  d_bits:
 * device uint32[ceil(n/32)] (bits past n are 0).  d_error: device float[n]
 * (16-byte aligned; may not alias d_x).  d_scale: device float[1].  With
 * n = 0 only *d_scale is written (0) and the other pointers may be NULL.
 * All work is queued on cuda_stream; the call does no cudaMalloc, cudaFree
 * or other allocating call.  Every call looks up the scratch array's
 * device address with the current device (a lookup, not an allocation);
 * the first call on a device also loads the library's device code there,
 * so make that first call before any stream capture.  Every call shares
 * the one scratch array and overwrites the part it reads, so calls that
 * overlap on the GPU (on different streams) race; serialize them.  n above
 * OB_STATIC_MAX_ELEMENTS returns OB_ERR_WORKSPACE; bad pointers
 * OB_ERR_INVALID_ARG / OB_ERR_ALIGN; a failed lookup or a failed launch of
 * this call's own kernels OB_ERR_CUDA (the call checks each launch's own
 * status; it does not read or clear an error left by earlier work). */
#define OB_STATIC_MAX_ELEMENTS ((int64_t)1 << 26)
OB_API ob_status ob_onebit_compress_static(const float *d_x, int64_t n, uint32_t *d_bits,
                                           float *d_error, float *d_scale, void *cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* ONEBIT_H */
