// mla.h -- launch interface of the MLA decode kernels (mla.cu), used by api.cu.
//
// MLA with absorbed weights ("MLA: multi-head latent attention", anrans.github.io
// attention-variants: weight absorption and decoupled RoPE): every query head scores one
// cached row per token, the 512-wide latent followed by the 64-wide RoPE key shared by all
// heads, and its output is the softmax-weighted sum of the rows' latent parts -- an MQA whose
// value is the first 512 entries of its key.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace gqa {

constexpr int kMlaLatent = 512;                   // d_c: latent width, also the value width
constexpr int kMlaRope = 64;                      // d_r: RoPE key width
constexpr int kMlaRow = kMlaLatent + kMlaRope;    // one cached row, one query row
constexpr int kMlaHeads = 16;                     // query heads per CTA
constexpr int kMlaTile = 32;                      // cached tokens per tile

struct MlaArgs {
    const __nv_bfloat16 *q;    // [B, Hq, 576]: absorbed latent query, then RoPE query
    const __nv_bfloat16 *kv;   // [B, Tmax, 576]: latent, then RoPE key
    const int32_t *seqlens;    // [B], device
    __nv_bfloat16 *out;        // [B, Hq, 512]
    float *part_o;             // [B, Hq, nsplit, 512] when nsplit > 1
    float *part_ml;            // [B, Hq, nsplit, 2] (running max in log2 units, weight sum)
    int B, Hq, Tmax, nsplit, chunk;
    float qscale;              // scale * log2(e)
};

struct MlaPlan {
    int nsplit;       // token ranges per sequence
    int chunk;        // tokens per range, a multiple of kMlaTile
    size_t ws_bytes;  // split partials (0 when nsplit == 1)
};

MlaPlan mla_plan_host(int B, int Hq, int Tmax, int num_sms);

// Enqueues the decode (and, for nsplit > 1, the combine) on `stream`; adds the launches made to
// *launches.  `before` / `after`, when non-null, are recorded around the decode kernel.
cudaError_t launch_mla_decode(const MlaArgs &a, cudaStream_t stream, int *launches, cudaEvent_t before,
                              cudaEvent_t after);

// The tensor-core MLA decode (mla_tc.cu): device-planned pieces, one persistent CTA per SM over
// (piece, 64-head block) units, a combine for split histories.  Workspace layout:
struct MlaTcPlan {
    int nsplit;       // most pieces one sequence can get
    int nhb;          // 64-head blocks
    size_t off_hdr, off_nsb, off_items, off_po, off_pml, ws_bytes;
};
// ws_budget bounds the split partials (fewer pieces per sequence when it is small).
MlaTcPlan mla_tc_plan_host(int B, int Hq, int Tmax, size_t ws_budget);

// Enqueues the planner, the decode and the combine on `stream` (three launches, added to
// *launches).  Tensor maps, all bf16 with the 128-byte swizzle:
//   tmKV2: kv_cache [B, Tmax, 576] viewed as (64 columns, Tmax, 9 column chunks, B), box {64, 128, 2, 1}
//          (two consecutive 128-token x 64-column chunk tiles);
//   tmKV1: kv_cache as (576, Tmax, B), box {64, 128, 1} (one chunk tile: the RoPE key);
//   tmQ:   q [B, Hq, 576] viewed as (64 columns, Hq, 9 column chunks, B), box {64, 64, 9, 1}.
// `before` / `after`, when non-null, are recorded around the decode kernel.
cudaError_t launch_mla_decode_tc(const CUtensorMap &tmKV2, const CUtensorMap &tmKV1, const CUtensorMap &tmQ,
                                 const void *q,
                                 const int32_t *seqlens, int B, int Hq, int Tmax, float scale, void *out, void *ws,
                                 const MlaTcPlan &p, int num_sms, int *status, unsigned long long wait_budget_ns,
                                 cudaStream_t stream, int *launches, cudaEvent_t before, cudaEvent_t after);

}  // namespace gqa
