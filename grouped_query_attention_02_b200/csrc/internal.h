// internal.h -- host-side interface between the C ABI (api.cu) and the kernel
// translation units (decode.cu, prefill.cu).  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gqa {

constexpr int kHeadDim = 128;       // the one head size this build implements
constexpr int kDecodeTile = 64;     // tokens per TMA stage of the CUDA-core decode kernel
constexpr int kDecodeCtasPerSm = 2; // resident CUDA-core decode CTAs per SM (shared-memory bound)
constexpr int kStatusTimeout = 6;   // device status word: a bounded wait gave up
constexpr int kStatusMisaligned = 3; // device status word: a kernel found its shared memory misaligned
// Caches of at most this many 128-token tiles (Tmax <= 512) take the tensor-core decode as one launch:
// whole histories as units, no planner and no combine, whose fixed costs would exceed what splitting
// a history this short could save.
constexpr int kStaticPlanTiles = 4;

struct DecodeArgs {
    const __nv_bfloat16 *q;   // [B,Hq,d]
    const int32_t *seqlens;   // [B], device
    __nv_bfloat16 *out;       // [B,Hq,d]
    float *part_o;            // [B,Hq,nsplit,d]   (nsplit > 1)
    float *part_ml;           // [B,Hq,nsplit,2]   (nsplit > 1)
    int *status;              // device status word
    int B, Hq, Hkv, Tmax, group, chunk, nsplit, nhb;
    float qscale;             // scale * log2(e)
    float qk_factor;          // FP8 cache: scale * log2(e) * k_scale
    float o_factor;           // FP8 cache: v_scale / 128 (the weights enter the PV product as 128 p)
    unsigned long long wait_budget_ns;
    // device-planned schedule (tensor-core path): see decode_tc.cu
    int *plan_hdr;            // {claim counter, pieces, C}
    int *nsplit_b;            // [B] pieces per sequence (the combine reads it when non-null)
    int4 *items;              // [B * nsplit] pieces, longest first
    int num_ctas;             // persistent CTAs (one per SM)
    // planner options for other operators that reuse decode_plan_kernel (0: the GQA decode's defaults)
    int out_row;              // output elements per (sequence, query head) row, zeroed for empty histories
    int plan_rounds;          // rounds of units per persistent CTA the pieces are sized for
    int static_plan;          // 1: no planner; one piece per history, units dealt round-robin (short caches)
    int tail_split;           // planner: a history's remainder is cut into up to this many pieces (0, 1: one)
};

// Host plan of a decode call and the layout of its workspace.
struct DecodePlan {
    int tile, chunk, nsplit, hb, nhb;
    bool tensor_cores;
    size_t off_hdr, off_nsb, off_items, off_po, off_pml, ws_bytes;
    bool static_plan;   // tensor-core path without the device planner: one launch, no workspace
};
// ws_budget bounds the split partials (fewer pieces per sequence when they would not fit; one piece needs none).
// fp8: the plan of the FP8-cache decode, which always takes the tensor-core path (group sizes <= 32).
DecodePlan decode_plan_host(int B, int Hq, int Hkv, int Tmax, int num_sms, size_t ws_budget, bool fp8 = false);

// Per-tensor scales of an FP8 (E4M3) cache: a key is e4m3(code) * k_scale, a value e4m3(code) * v_scale.
struct Fp8Scales {
    float k_scale, v_scale;
};

// Enqueues one decode (all kernels) on `stream` with the workspace `ws` laid out by `p`; `fp8` non-null:
// the caches hold E4M3 codes with those scales (p must then come from decode_plan_host(..., true)).
// Returns 0 or a gqa_status code; adds the kernels launched to *launches.
int decode_enqueue(const void *q, const void *k, const void *v, const int32_t *seqlens, int B, int Hq, int Hkv,
                   int Tmax, float scale, void *out, void *ws, const DecodePlan &p, int num_sms, int *status,
                   cudaStream_t stream, int *launches, cudaEvent_t ev_before, cudaEvent_t ev_after,
                   const Fp8Scales *fp8 = nullptr);

// How the decode of group size g is laid out: the kernel family (tensor cores for
// 3 <= g <= 32, CUDA cores otherwise), its token tile (TMA box rows and split
// granularity), query heads per CTA, CTAs per SM for the split planner.
struct DecodeShape {
    bool tensor_cores;
    int tile;          // tokens per pipeline stage
    int heads_per_cta; // query heads one CTA serves
    int nhb;           // CTAs per (sequence, KV head, split)
    int ctas_per_sm;
};
DecodeShape decode_shape(int g);
int decode_heads_per_cta(int g);   // CUDA-core kernel only

// Launches the CUDA-core decode kernel (group sizes outside the tensor-core range).
cudaError_t launch_decode_split(const CUtensorMap &tmK, const CUtensorMap &tmV, const DecodeArgs &a,
                                cudaStream_t stream);
// fp8: tmK / tmV map E4M3 code tiles (128 tokens x 128 bytes) instead of bf16 halves.
cudaError_t launch_decode_tc(const CUtensorMap &tmK, const CUtensorMap &tmV, const CUtensorMap &tmQ,
                             const DecodeArgs &a, cudaStream_t stream, bool fp8);
cudaError_t launch_decode_plan(const DecodeArgs &a, cudaStream_t stream);
// pdl: launched as a programmatic dependent of the previous kernel on the stream
cudaError_t launch_decode_combine(const DecodeArgs &a, cudaStream_t stream, bool pdl = false);
cudaError_t launch_repeat_kv(const void *k, const void *v, const int32_t *seqlens, void *k_rep, void *v_rep,
                             int B, int Tmax, int Hq, int Hkv, cudaStream_t stream);
cudaError_t launch_wait_timeout_selftest(int *status, unsigned long long budget_ns, cudaStream_t stream);

struct PrefillArgs {
    __nv_bfloat16 *out;       // [B,S,Hq,d]
    float *lse;               // [B,Hq,S] natural log-sum-exp of each row's scaled scores, or null
    int *status;
    int B, S, Hq, Hkv, group;
    float qscale;             // log2(e) / sqrt(d)
    unsigned long long wait_budget_ns;
};

// Causal prefill backward (backward.cu): D = rowsum(dO * O), then dK/dV per key tile (summed over the
// group's heads), then dQ per query tile.
struct BackwardArgs {
    const __nv_bfloat16 *out, *dout;   // [B,S,Hq,d]
    const float *lse;                  // [B,Hq,S] natural log-sum-exp from the forward
    float *dsum;                       // [B,Hq,S] workspace: D = rowsum(dO * O)
    __nv_bfloat16 *dq;                 // [B,S,Hq,d]
    __nv_bfloat16 *dk, *dv;            // [B,S,Hkv,d]
    int *status;
    int B, S, Hq, Hkv, group;
    float qscale;                      // log2(e) / sqrt(d)
    float scale;                       // 1 / sqrt(d)
    unsigned long long wait_budget_ns;
};
cudaError_t launch_prefill_backward(const CUtensorMap &tmQ, const CUtensorMap &tmK, const CUtensorMap &tmV,
                                    const CUtensorMap &tmDO, const BackwardArgs &a, cudaStream_t stream,
                                    int *launches);

// The current device's status word (address of the library's device variable), or null.
int *device_status_word();
// Sets what gqa_last_launch_count() reports on this host thread.
void set_last_launch_count(int n);

cudaError_t launch_prefill(const CUtensorMap &tmQ, const CUtensorMap &tmK, const CUtensorMap &tmV,
                           const PrefillArgs &a, cudaStream_t stream);

}  // namespace gqa
