// onebit_kernels.cuh -- device code of libonebit (sm_100a).
//
// The compression-phase step of 1-bit Adam ("1-bit Adam: Communication
// Efficient Large-Scale Training with Adam's Convergence Speed", review
// page, sections "Abstract" and "Proposed method") as five HBM-streaming
// launches over a list of 4096-element tiles, each launched so that it may
// start while the one before it finishes (programmatic dependent launch):
//
//   ob_pack_kernel          worker stage, all W workers of a tile per CTA
//   ob_scale_kernel         the worker scales from the per-tile sums
//   ob_server_kernel        server stage of a tile (the first 8 workers'
//                           sequential sums from a per-tile table)
//   ob_scale_kernel         the server scales from the per-tile sums
//   ob_apply_kernel         gather, decode, preconditioned update
//
// plus the warmup Adam step, the freeze and an error decoder used when the
// host reads state, and the 1-bit LAMB variants (kernels/lamb.cuh: the
// warmup in two passes, the norms, the update with layerwise rates).  No
// step is a dense contraction, so no tensor cores: every kernel is a stream
// of coalesced 16- or 32-byte loads and stores, bound by HBM bandwidth.
//
// Numerics.  Every fp32 operation is written with an explicit
// round-to-nearest intrinsic (__fmul_rn, __fadd_rn, __fsub_rn, __fdiv_rn,
// __fsqrt_rn), so nvcc cannot contract a*b+c into an FMA, and the order of
// operations is the method's: the results are the same IEEE binary32
// values a plain sequential CPU evaluation gives.  Sums of squares for the
// scales are taken in fp64 in a fixed order (per thread, warp butterfly,
// warps in order, tiles in order), so results repeat run to run.
//
// Lazy error buffers.  e_w = x - sign(x) s_w needs s_w, which needs all of
// x.  Rather than a second pass over x, the worker error is stored as the
// pair (x, s_w) and decoded where it is next used:
//   e_w = fl(x - sign(x) s_w)   -- the same rounding an eager pass would do.
// The server error is stored the same way as (y, s'_j).
#pragma once

#include "kernels/common.cuh"
#include "kernels/warmup.cuh"
#include "kernels/pack.cuh"
#include "kernels/scale.cuh"
#include "kernels/server.cuh"
#include "kernels/apply.cuh"
#include "kernels/lamb.cuh"
#include "kernels/state.cuh"
#include "kernels/compress_static.cuh"
