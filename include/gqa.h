/*
 * gqa.h -- C ABI of libgqa.so: grouped-query attention (GQA) on one B200.
 *
 * The operator.  Hq query heads are split into Hkv consecutive groups of
 * g = Hq / Hkv heads; query head h reads KV head h / g.  Hq must be a
 * multiple of Hkv.  MHA (Hkv == Hq) and MQA (Hkv == 1) are the two ends of
 * the same operator.  Definitions: study.greatitself.com "grouped-query and
 * multi-query attention" (mapping paragraph); lihaoran.work/?p=2890 "Shared KV
 * can still produce different outputs" (each query head keeps its own
 * softmax(q K^T / sqrt(d)) V); anrans.github.io attention-variants "Kernels do
 * not need to copy the KV heads" (a group's query heads read one shared KV
 * head, read once, never copied; causal mask as a lower triangle).
 *
 * Conventions shared by every entry point.
 *  - Tensors are bf16 (IEEE binary32 with the low 16 bits dropped), except the
 *    one-byte E4M3 caches of gqa_decode_fp8, dense and row-major in the layouts
 *    named below; all device pointers must be 16-byte aligned.  Accumulation
 *    is fp32; outputs are rounded to bf16.
 *  - `stream` is a cudaStream_t passed as void*; NULL means the legacy
 *    default stream.  Every call only enqueues work on `stream` and returns;
 *    no call synchronises the host, and the caller owns every tensor and the
 *    stream.  Results are ready when the stream has reached them.
 *  - Host-side argument checks run before anything is enqueued; a failed
 *    check returns its status and enqueues nothing.  A CUDA launch error is
 *    returned as GQA_ERR_CUDA.
 *  - The library keeps, per device, a grow-only workspace for the split-KV
 *    plan and partial results (allocated on first need with cudaMalloc, or
 *    by the caller's allocator: gqa_set_workspace_allocator);
 *    gqa_release() frees it.  TMA tensor maps are encoded on the host for
 *    every call (kernel parameters, nothing is cached).  Calls that share the
 *    workspace on one device must be ordered on one stream (or otherwise
 *    serialised by the caller).
 *  - Only head_dim d == 128 is implemented (GQA_ERR_UNSUPPORTED otherwise).
 */
#ifndef GQA_H_
#define GQA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gqa_status {
    GQA_OK = 0,
    GQA_ERR_INVALID_ARG = 1,    /* null pointer, non-positive size, Hq % Hkv != 0 */
    GQA_ERR_UNSUPPORTED = 2,    /* a valid shape this build does not implement (d != 128) */
    GQA_ERR_MISALIGNED = 3,     /* a pointer not 16-byte aligned */
    GQA_ERR_OUT_OF_MEMORY = 4,  /* the workspace could not be allocated */
    GQA_ERR_CUDA = 5,           /* a CUDA runtime/driver call or launch failed */
    GQA_ERR_DEVICE_TIMEOUT = 6  /* a kernel gave up a bounded wait (read by gqa_get_last_device_status) */
} gqa_status;

/*
 * gqa_decode -- one decode step over a bf16 KV cache.
 *
 *   q        [B, Hq, d]        the step's query, one row per (sequence, query head)
 *   k_cache  [B, Tmax, Hkv, d] keys of every cached token (the step's own token included)
 *   v_cache  [B, Tmax, Hkv, d] values, same layout
 *   seqlens  [B] int32, DEVICE memory: cached tokens of each sequence
 *   scale    multiplier of q.k (normally 1/sqrt(d))
 *   out      [B, Hq, d]        out[b,h] = sum_{t < seqlens[b]} softmax_t(scale q[b,h].k[b,t,h/g]) v[b,t,h/g]
 *
 * Sequence b attends to every cached token t < seqlens[b]; rows at or past
 * seqlens[b] are never used (they may hold anything, NaN included).
 * Preconditions not checked on the host (checking needs a device read):
 * 0 <= seqlens[b] <= Tmax; values outside are clamped to [0, Tmax].  A
 * sequence with seqlens[b] == 0 gets an all-zero output row.  A NaN inside
 * the history follows the definition: a NaN key makes the outputs of every
 * head of its group NaN, a NaN value element makes that output coordinate
 * NaN for the group's heads.
 *
 * Each K/V tile is fetched once by TMA and shared by the g query heads of its
 * group.  For 3 <= g <= 32 the products run on the tcgen05 tensor cores and
 * the histories are cut into pieces on the device from the actual lengths
 * (longest first), processed by one persistent CTA per SM; pieces of one
 * history are merged by a log-sum-exp combine kernel.  Other group sizes use
 * a CUDA-core kernel with a host-side split.  Either way the work goes
 * through the library workspace.
 */
gqa_status gqa_decode(const void *q, const void *k_cache, const void *v_cache, const int32_t *seqlens,
                      int B, int Hq, int Hkv, int d, int Tmax, float scale, void *out, void *stream);

/*
 * gqa_decode_fp8 -- one decode step over an FP8 (E4M3) KV cache with
 * per-tensor scales, the cache quantisation that "Other ways to shrink the KV
 * cache" (anrans.github.io attention-variants) lists: K and V stored in FP8,
 * half the bytes of bf16.
 *
 *   q        [B, Hq, d]        bf16, as in gqa_decode
 *   k_cache  [B, Tmax, Hkv, d] one-byte E4M3 codes (the "fn" variant: no
 *                              infinities, 0x7F / 0xFF are NaN, largest finite 448)
 *   v_cache  [B, Tmax, Hkv, d] E4M3 codes, same layout
 *   k_scale, v_scale           a key element is e4m3(code) * k_scale, a value
 *                              element e4m3(code) * v_scale (finite floats)
 *   seqlens, scale, out, stream: as in gqa_decode
 *
 *   out[b,h] = sum_{t < seqlens[b]} softmax_t(scale q[b,h].K[b,t,h/g]) V[b,t,h/g]
 *   with K = e4m3(k_cache) * k_scale and V = e4m3(v_cache) * v_scale.
 *
 * Group sizes g = Hq / Hkv up to 32 (GQA_ERR_UNSUPPORTED above).  Each tile
 * is read once by TMA.  The scores are E4M3 tensor-core products straight
 * from the key codes, with the query as two E4M3 terms of q 2^e per head:
 * every query element down to 2^-10 of its head's largest |q| is carried
 * exactly, smaller ones within 2^-17 of that largest.  The value codes are
 * widened to f16 on the SM, exactly, and the softmax weights enter the P.V
 * product as f16 values of 128 p (relative rounding at most 2^-11 per weight;
 * the normalising sum is taken in fp32); every product accumulates in fp32.  NaN codes inside the history
 * propagate to the output; rows past seqlens[b] are never used.  Same
 * workspace, stream and error rules as gqa_decode.
 */
gqa_status gqa_decode_fp8(const void *q, const void *k_cache, const void *v_cache, const int32_t *seqlens, int B,
                          int Hq, int Hkv, int d, int Tmax, float scale, float k_scale, float v_scale, void *out,
                          void *stream);

/*
 * gqa_decode_noalloc -- gqa_decode for callers that cannot let a library
 * allocate device memory.  (This entry point is an engineering addition; the
 * pages describe no counterpart.)
 *
 * Who needs it: a serving engine that reserves nearly all of the GPU for its
 * own memory pool (typically to size its KV cache) has nothing left for a
 * library's cudaMalloc, and a latency-critical decode loop cannot absorb
 * cudaMalloc's implicit synchronisation and unpredictable cost.  This call
 * allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 *
 * Arguments, layouts, result and the other error codes are those of
 * gqa_decode; the caller still owns and passes every input and output.  The
 * split-KV partials go to a fixed 32 MiB array compiled into the library,
 * which every GPU that loads the library holds until the process exits.
 *  - The split plan is gqa_decode's with the pieces per sequence reduced
 *    until the workspace (split partials of about B*Hq*nsplit*(d+2)*4 bytes
 *    plus the piece list) fits; returns GQA_ERR_UNSUPPORTED when even one
 *    piece per sequence does not fit 32 MiB (B*Hq*(d+2)*4 bytes > 32 MiB);
 *    gqa_decode handles such shapes.
 *  - The first call on a device looks up the array's device address once,
 *    with that device current; make that first call before any stream
 *    capture.
 *  - Every call on a device shares the one array and it keeps the last
 *    call's contents; nothing in it needs to start at zero because each call
 *    writes every partial it later reads.  Calls whose kernels overlap on the
 *    GPU (different streams, no ordering between them) race on the array and
 *    give wrong results: order them, e.g. on one stream.
 */
gqa_status gqa_decode_noalloc(const void *q, const void *k_cache, const void *v_cache, const int32_t *seqlens,
                              int B, int Hq, int Hkv, int d, int Tmax, float scale, void *out, void *stream);

/*
 * gqa_prefill_causal -- causal self-attention over whole prompts.
 *
 *   q    [B, S, Hq, d]
 *   k, v [B, S, Hkv, d]
 *   out  [B, S, Hq, d]   out[b,r,h] = sum_{t <= r} softmax_t(q[b,r,h].k[b,t,h/g] / sqrt(d)) v[b,t,h/g]
 *
 * Row r sees tokens 0..r (lower triangle including the diagonal); the scale
 * is 1/sqrt(d).  QK^T and PV run on the tcgen05 tensor cores with fp32
 * accumulators in tensor memory; the softmax weights are rounded to bf16
 * before the PV product.  No workspace.
 */
gqa_status gqa_prefill_causal(const void *q, const void *k, const void *v, int B, int S, int Hq, int Hkv,
                              int d, void *out, void *stream);

/*
 * gqa_prefill_causal_fwd -- gqa_prefill_causal that also returns, per query
 * row, the log-sum-exp of its scaled scores, which the backward needs:
 *
 *   lse  [B, Hq, S] fp32, device: lse[b,h,r] = log sum_{t <= r} exp(q[b,r,h].k[b,t,h/g] / sqrt(d))
 *        (natural log; 4-byte aligned)
 *
 * out as in gqa_prefill_causal.
 */
gqa_status gqa_prefill_causal_fwd(const void *q, const void *k, const void *v, int B, int S, int Hq, int Hkv,
                                  int d, void *out, float *lse, void *stream);

/*
 * gqa_prefill_causal_bwd -- gradients of a loss through gqa_prefill_causal.
 * During training a shared key or value head receives the gradient of every
 * query head of its group (study.greatitself.com "grouped-query and
 * multi-query attention", training paragraph); dk and dv are those sums.
 *
 *   q, k, v, out, lse  the forward's inputs, output and log-sum-exp (gqa_prefill_causal_fwd)
 *   dout  [B, S, Hq, d]   dL/dout
 *   dq    [B, S, Hq, d]   dL/dq, written
 *   dk, dv [B, S, Hkv, d] dL/dk, dL/dv, written (each the sum over the group's query heads)
 *
 * With P = exp(q.k / sqrt(d) - lse) (causal), dP = dout v^T, D = rowsum(dout * out),
 * dS = P (dP - D): dv = sum_h P^T dout, dk = sum_h dS^T q / sqrt(d), dq = dS k / sqrt(d).
 * P and dS are rounded to bf16 for the tensor-core products (fp32 accumulation); D is
 * computed from the bf16 out.  Uses B*Hq*S*4 bytes of the library workspace; two
 * kernels (dq, which also forms D, then dk/dv).  Same layouts, alignment and error rules as
 * gqa_prefill_causal.
 */
gqa_status gqa_prefill_causal_bwd(const void *q, const void *k, const void *v, const void *out, const float *lse,
                                  const void *dout, int B, int S, int Hq, int Hkv, int d, void *dq, void *dk,
                                  void *dv, void *stream);

/*
 * gqa_decode_expanded -- the same decode computed the wasteful way, kept as a
 * baseline: every KV head is first physically repeated g times into the
 * caller's buffers k_rep/v_rep [B, Tmax, Hq, d] (rows t < seqlens[b] are
 * written, the rest untouched), then the decode kernel runs with one query
 * head per KV head.  Same arguments and result as gqa_decode; the buffers
 * must each hold gqa_decode_expanded_bytes(B, Tmax, Hq, d) bytes.
 */
gqa_status gqa_decode_expanded(const void *q, const void *k_cache, const void *v_cache, const int32_t *seqlens,
                               int B, int Hq, int Hkv, int d, int Tmax, float scale, void *out,
                               void *k_rep, void *v_rep, void *stream);

/* Bytes of ONE repeated cache (k_rep or v_rep) for gqa_decode_expanded; 0 on bad sizes. */
size_t gqa_decode_expanded_bytes(int B, int Tmax, int Hq, int d);

/*
 * gqa_decode_plan -- the split-KV plan gqa_decode uses, for a device with
 * num_sms SMs: tokens per split (*chunk, a multiple of the kernel's token
 * tile), number of splits (*nsplit) and workspace bytes it needs
 * (*workspace_bytes).  For group sizes 3..32 (the tensor-core kernel) the
 * histories are cut on the device from the actual lengths: *chunk is then the
 * smallest piece and *nsplit the most pieces one sequence can get, and the
 * workspace also holds the piece list.  Pure host arithmetic; touches no device.
 */
gqa_status gqa_decode_plan(int B, int Hq, int Hkv, int d, int Tmax, int num_sms, int *chunk, int *nsplit,
                           size_t *workspace_bytes);

/*
 * gqa_mla_decode -- one decode step of multi-head latent attention with
 * absorbed weights ("MLA: multi-head latent attention", anrans.github.io
 * attention-variants: weight absorption and decoupled RoPE).  The cache holds
 * one row per token, the d_c-wide latent followed by the d_r-wide RoPE key
 * shared by all heads; the latent is both key and value, so the operator is an
 * MQA whose value is the first d_c entries of its key.
 *
 *   q        [B, Hq, d_c + d_r]   per head: the absorbed latent query (W_UK
 *                                 folded in), then the RoPE query
 *   kv_cache [B, Tmax, d_c + d_r] per token: latent, then RoPE key
 *   seqlens  [B] int32, DEVICE memory
 *   scale    multiplier of q.kv (the original head's 1/sqrt(d_h + d_r))
 *   out      [B, Hq, d_c]         out[b,h] = sum_{t < seqlens[b]}
 *                                 softmax_t(scale q[b,h].kv[b,t]) kv[b,t,0:d_c]
 *                                 (W_UV is applied by the caller's output projection)
 *
 * bf16 in and out, fp32 accumulation; d_c = 512 and d_r = 64 only
 * (GQA_ERR_UNSUPPORTED otherwise); B and Hq at most 65535; q, kv_cache and out
 * 16-byte aligned, seqlens 4-byte aligned (GQA_ERR_MISALIGNED otherwise).
 * Lengths, NaN and empty histories as in gqa_decode.
 *
 * Runs on the tcgen05 tensor cores: blocks of 64 query heads, tokens as the
 * 128-row side of S^T = KV.Q^T and of O^T += KV_latent^T.P^T, the cached rows
 * fetched by TMA once per head block; histories are cut into pieces on the
 * device from the real lengths and merged by a combine kernel, through the
 * library workspace (three launches: plan, decode, combine).  The weights
 * enter the P.V product rounded to bf16, as in the causal prefill, so each
 * output is a convex combination of latent rows with weights within 2^-8 of
 * the exact ones.
 */
gqa_status gqa_mla_decode(const void *q, const void *kv_cache, const int32_t *seqlens, int B, int Hq, int d_c,
                          int d_r, int Tmax, float scale, void *out, void *stream);

/*
 * gqa_mla_decode_cudacore -- the same operator as gqa_mla_decode, same
 * arguments, checks and errors, computed on the CUDA cores (16 heads per CTA,
 * tiles of 32 cached rows through shared memory, fp32 weights and dot
 * products, split over token ranges and merged by a combine kernel through the
 * library workspace).  About two orders of magnitude slower; it is kept as an
 * independent second path that full-size outputs of the tensor-core kernel can
 * be compared with where the fp64 oracle would take too long.
 */
gqa_status gqa_mla_decode_cudacore(const void *q, const void *kv_cache, const int32_t *seqlens, int B, int Hq,
                                   int d_c, int d_r, int Tmax, float scale, void *out, void *stream);

/*
 * gqa_tp_shard -- the heads rank `rank` of `tp` tensor-parallel ranks owns
 * for one attention layer (kv-head-replication glossary entry,
 * inferencex.semianalysis.com; the tensor-parallelism paragraphs of
 * deepconcepts.dev Grouped-Query Attention).  Ranks own consecutive, equal
 * runs of query heads: [*q_first, *q_first + *q_count), Hq / tp each.
 *  - Hkv >= tp (Hkv a multiple of tp): the KV heads are partitioned, Hkv / tp
 *    per rank, [*kv_first, *kv_first + *kv_count), exactly the groups of the
 *    rank's query heads.
 *  - Hkv < tp (tp a multiple of Hkv): a rank's query heads lie in one group;
 *    the rank keeps its own replica of that group's KV head (*kv_count = 1),
 *    tp / Hkv ranks holding the same one.
 * The rank then runs gqa_decode (or gqa_decode_fp8) on its shard: q
 * [B, *q_count, d] and caches [B, Tmax, *kv_count, d], whose local group size
 * is *q_count / *kv_count.  No exchange is needed inside attention; the
 * output projection that follows is row-parallel over the same heads.
 * GQA_ERR_INVALID_ARG for null pointers, non-positive sizes, rank outside
 * [0, tp) or Hq % Hkv != 0; GQA_ERR_UNSUPPORTED when Hq % tp != 0 or neither
 * of Hkv, tp divides the other.  Pure host arithmetic; touches no device.
 */
gqa_status gqa_tp_shard(int Hq, int Hkv, int tp, int rank, int *q_first, int *q_count, int *kv_first,
                        int *kv_count);

/*
 * gqa_get_last_device_status -- synchronises `stream`, then reads and clears
 * the device's status word.  Kernels never trap: a kernel that gives up a
 * bounded wait (about a second) records GQA_ERR_DEVICE_TIMEOUT there and
 * returns; one that finds its shared-memory window not 1024-byte aligned
 * (which the 128-byte swizzle needs) records GQA_ERR_MISALIGNED and does
 * nothing.  Returns GQA_OK when nothing was recorded, GQA_ERR_CUDA when the
 * synchronisation itself failed.
 */
gqa_status gqa_get_last_device_status(void *stream);

/*
 * gqa_selftest_wait_timeout -- enqueues one tiny kernel that waits on a
 * shared-memory barrier nothing will ever complete, bounded to about
 * timeout_us microseconds, and records GQA_ERR_DEVICE_TIMEOUT.  Used by the
 * tests to show that a stuck wait returns instead of hanging the GPU.
 */
gqa_status gqa_selftest_wait_timeout(int timeout_us, void *stream);

/*
 * gqa_set_profile_events -- measurement hook.  When both are non-NULL
 * (cudaEvent_t passed as void*), every later gqa_decode / gqa_decode_fp8 /
 * gqa_mla_decode / gqa_prefill_causal(_fwd) / gqa_decode_expanded records `before` on its stream
 * immediately before its dominant kernel (the decode kernel; the prefill
 * kernel) and `after` immediately after it; gqa_prefill_causal_bwd records
 * them around its two kernels; gqa_decode_noalloc records nothing.  NULL,
 * NULL turns the hook off.
 */
gqa_status gqa_set_profile_events(void *before, void *after);

/* Number of kernels the most recent call on this host thread enqueued. */
int gqa_last_launch_count(void);

/* Frees (hands back to its allocator) the workspace of every device the
 * library used.  Call it with no library work in flight. */
void gqa_release(void);

/*
 * gqa_set_workspace_allocator -- where the per-device workspace comes from.
 * By default it is cudaMalloc'd on first need and grown, never shrunk, as
 * calls need more; an engine that already owns the GPU's memory can hand the
 * library blocks from its own pool instead.
 *
 *   alloc(bytes, device, ctx)          a block of at least `bytes` bytes of
 *                                      device memory on `device`, 256-byte
 *                                      aligned, or NULL when there is none
 *   free_fn(ptr, bytes, device, ctx)   takes back a block alloc returned
 *                                      (`bytes` as requested)
 *   ctx                                passed through to both
 *
 * Both NULL restores cudaMalloc / cudaFree; exactly one NULL is
 * GQA_ERR_INVALID_ARG.  The call first hands every current workspace back to
 * the allocator that made it, so, like gqa_release, it must run with no
 * library work in flight.  When alloc returns NULL, the call that needed the
 * workspace returns GQA_ERR_OUT_OF_MEMORY with nothing enqueued; a block that
 * is not 256-byte aligned is handed back and that call returns
 * GQA_ERR_MISALIGNED.  Before free_fn receives a block the library
 * synchronises the block's device (as cudaFree does), so no enqueued kernel
 * still reads it.  Both functions run with the library's lock held, with the
 * block's device current, and must not call back into the library.
 */
typedef void *(*gqa_alloc_fn)(size_t bytes, int device, void *ctx);
typedef void (*gqa_free_fn)(void *ptr, size_t bytes, int device, void *ctx);
gqa_status gqa_set_workspace_allocator(gqa_alloc_fn alloc, gqa_free_fn free_fn, void *ctx);

/* Text for a status code (static storage). */
const char *gqa_status_string(gqa_status status);

/* Library version, e.g. "gqa-b200 0.1". */
const char *gqa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GQA_H_ */
