// mla_tc.cu -- MLA decode with absorbed weights on the tcgen05 tensor cores.
//
// The operator ("MLA: multi-head latent attention", anrans.github.io attention-variants, weight
// absorption and decoupled RoPE): every query head scores one shared cached row per token, the
// 512-wide latent followed by the 64-wide RoPE key, and its output is the softmax-weighted sum of
// the rows' latent parts.  Per cached token that is 2 x Hq x (576 + 512) FLOP against 1152 bytes,
// about 242 FLOP per byte at 128 heads: a dense contraction, close to the B200's ridge point.
//
// One CTA serves a block of 64 query heads of one sequence over a piece of its history, with the
// tokens as the 128-row M side of both products:
//
//   S^T [128 tokens x 64 heads]   = KV_tile [128 x 576] . Q_blk^T        (A = KV, K-major; B = Q, K-major)
//   O^T [512 latent x 64 heads]  += KV_tile[:, 0:512]^T . P^T [128 x 64]  (A = latent, MN-major; B = P^T)
//
// O^T takes 4 blocks x 64 = 256 of the 512 tensor-memory columns and S^T another 64; a block of
// all 128 heads would need all 512 for O^T alone, so the two head blocks of a DeepSeek-shaped
// decode are two units whose CTAs read the same tiles (the second read is normally served by L2).
//
// Shared memory holds the block's query rows (9 chunks of 64 heads x 64 columns, 72 KB) and one
// tile as 9 column chunks of 128 tokens x 64 columns (16 KB each, 128-byte swizzle): chunks 0..7
// are the latent, read twice -- as K rows by the S^T product and as V^T by the PV product, so the
// latent crosses HBM once -- and chunk 8 is the RoPE key.  Once S^T is done the RoPE chunk is free
// and holds the weights P^T; the PV product frees the latent chunks two at a time (one 128-row
// block of O^T each), and the next tile's chunks stream into them while the rest of the PV runs.
//
// The weights enter the PV product rounded to bf16 (as in the causal prefill); the weight sum is
// taken over the same rounded values, so the output is an exact convex combination of the latent
// rows with weights within 2^-8 of the exact ones.
//
// Scheduling is the GQA decode's: decode_plan_kernel cuts the histories into pieces from the real
// lengths (sized for about two rounds of units per CTA: a unit's query rows and its 128 KB of
// partials are a fixed cost), one persistent CTA per SM claims (piece, head block) units, and
// mla_combine_planned_kernel merges the pieces of split histories.  All three are chained with
// programmatic dependent launch.
//
// Warps: 0..15 softmax and epilogue (four warpgroups of 16 heads; thread = token of S^T, latent
// row of O^T), 16 the TMA producer (it also claims units), 17 the tensor-memory allocator and MMA
// issuer, 18 an L2 prefetcher, 19 a second TMA issuer.  Every wait is bounded and reports a timeout
// through the device status word.
#include "internal.h"
#include "mla.h"
#include "ptx.cuh"

namespace gqa {
namespace {

constexpr int kTok = 128;                         // tokens per tile (M of S^T)
constexpr int kNh = 64;                           // query heads per CTA (N of both products)
constexpr int kChunks = kMlaRow / 64;             // 9 column chunks of 64 per row
constexpr int kLatChunks = kMlaLatent / 64;       // 8 of them latent
constexpr int kRopeSlot = kLatChunks;             // the RoPE chunk's slot, then P^T's
constexpr int kChunkBytes = kTok * 128;           // 16 KB: one chunk of a tile
constexpr int kQChunkBytes = kNh * 128;           // 8 KB: one chunk of the block's query rows
constexpr int kWG = 128;
constexpr int kNWG = 4;                           // softmax / epilogue warpgroups
constexpr int kHW = kNh / kNWG;                   // heads per warpgroup (16)
constexpr int kProducerWarp = 4 * kNWG;
constexpr int kMmaWarp = kProducerWarp + 1;
constexpr int kPrefetchWarp = kMmaWarp + 1;       // keeps the tiles kAhead ahead of the producer in L2
// A second TMA issuer: one thread completes about one box per 300 ns whatever its size, so the odd latent
// chunk pairs of every tile come from this warp while the producer issues the even ones and the RoPE chunk
constexpr int kCoProducerWarp = kPrefetchWarp + 1;
constexpr int kThreads = kWG * kNWG + 128;
constexpr int kAhead = 2;
constexpr int kQD = 4;                            // depth of the unit queue
constexpr float kMoveThreshold = 8.0f;            // the running maximum moves only by more than this
constexpr int kGroups = kLatChunks / 2 + 1;       // loads per tile: four latent chunk pairs, then the RoPE chunk

// barrier slots
enum : int { CH_FULL = 0, EMPTY_PAIR = CH_FULL + kGroups, EMPTY_P = EMPTY_PAIR + kLatChunks / 2, S_FULL, P_FULL,
             Q_FULL, Q_EMPTY, O_FULL, O_FREE, I_FULL, I_EMPTY = I_FULL + kQD, DRAIN = I_EMPTY + kQD, GRP,
             kBars = GRP + kNWG };

// shared-memory layout (bytes)
constexpr int kSlotOff = 0;                                  // 9 tile chunks
constexpr int kQOff = kSlotOff + kChunks * kChunkBytes;      // 9 query chunks
constexpr int kRedOff = kQOff + kChunks * kQChunkBytes;      // [2][4][64] floats: tile maxima per warp
constexpr int kLsumOff = kRedOff + 2 * 4 * kNh * 4;          // [4][64] floats: weight sums per warp
constexpr int kVoteOff = kLsumOff + 4 * kNh * 4;             // [2 wg][2][4] ints
constexpr int kQueueOff = kVoteOff + kNWG * 8 * 4;           // kQD units of 8 ints
constexpr int kBarOff = kQueueOff + kQD * 32;
constexpr int kTmemOff = kBarOff + kBars * 8;
constexpr int kErrOff = kTmemOff + 8;
constexpr int kIssuedOff = kErrOff + 4;                      // tiles the producer has issued (for the prefetcher)
constexpr int kSmemBytes = kErrOff + 8;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
static_assert(kNh * kTok * 2 == kChunkBytes, "P^T fills the RoPE chunk's slot exactly");

// tensor memory: O^T blocks j = 0..3 at columns 64 j, S^T at 256
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCol = 4 * kNh;
static_assert(kSCol + kNh <= kTmemCols, "tensor-memory budget");

struct MlaTcArgs {
    __nv_bfloat16 *out;        // [B, Hq, 512]
    float *part_o;             // [B, Hq, nsplit, 512]
    float *part_ml;            // [B, Hq, nsplit, 2]
    int *status;
    const int *plan_hdr;       // {claim counter, pieces, C}
    int *claim;                // = plan_hdr (the claim counter)
    const int *nsplit_b;       // [B] pieces per sequence
    const int4 *items;         // pieces {b, piece, t_begin, t_end}, longest first
    int B, Hq, nsplit, nhb;
    float qscale;              // scale * log2(e)
    unsigned long long wait_budget_ns;
};

__device__ __forceinline__ void record_status(int *status, int code)
{
    if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ bool wait_or_fail(uint64_t *bar, uint32_t parity, const MlaTcArgs &a, volatile int *err)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*err) return false;
        if (global_timer_ns() - t0 > a.wait_budget_ns) {
            *err = 1;
            record_status(a.status, kStatusTimeout);
            return false;
        }
    }
    return true;
}

// Barrier among one warpgroup's 128 threads on an mbarrier (bounded like every other wait).
__device__ __forceinline__ bool group_sync(uint64_t *grp, int &uses, const MlaTcArgs &a, volatile int *err)
{
    mbar_arrive(grp);
    const bool r = wait_or_fail(grp, uses & 1, a, err);
    ++uses;
    return r;
}

// kHW consecutive tensor-memory columns per thread (16 or 32)
__device__ __forceinline__ void tmem_ld_hw(uint32_t taddr, uint32_t (&r)[kHW])
{
    if constexpr (kHW == 16) tmem_ld16(taddr, r);
    else tmem_ld32(taddr, r);
}
__device__ __forceinline__ void tmem_st_hw(uint32_t taddr, const uint32_t (&r)[kHW])
{
    if constexpr (kHW == 16) tmem_st16(taddr, r);
    else tmem_st32(taddr, r);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__global__ void __launch_bounds__(kThreads, 1)
mla_decode_tc_kernel(const __grid_constant__ CUtensorMap tmKV2, const __grid_constant__ CUtensorMap tmKV1,
                     const __grid_constant__ CUtensorMap tmQ, const MlaTcArgs a)
{
    // the 128-byte swizzle needs 1024-byte aligned chunks; a misaligned window is reported
    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) record_status(a.status, kStatusMisaligned);
        return;
    }
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + kBarOff);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kTmemOff);
    volatile int *err = reinterpret_cast<volatile int *>(smem + kErrOff);
    volatile int *queue = reinterpret_cast<volatile int *>(smem + kQueueOff);

    if (threadIdx.x == 0) {
        for (int g = 0; g < kGroups; ++g) mbar_init(&bar[CH_FULL + g], 1);
        for (int j = 0; j < kLatChunks / 2; ++j) mbar_init(&bar[EMPTY_PAIR + j], 1);
        mbar_init(&bar[EMPTY_P], 1);
        mbar_init(&bar[S_FULL], 1);
        mbar_init(&bar[P_FULL], kWG * kNWG);
        mbar_init(&bar[Q_FULL], 1);
        mbar_init(&bar[Q_EMPTY], 1);
        mbar_init(&bar[O_FULL], 1);
        mbar_init(&bar[O_FREE], kWG * kNWG);
        for (int s = 0; s < kQD; ++s) {
            mbar_init(&bar[I_FULL + s], 1);
            mbar_init(&bar[I_EMPTY + s], 3 + kWG * kNWG);   // MMA issuer, prefetcher, co-producer, softmax threads
        }
        mbar_init(&bar[DRAIN], 1);
        for (int w = 0; w < kNWG; ++w) mbar_init(&bar[GRP + w], kWG);
        *err = 0;
        *reinterpret_cast<volatile int *>(smem + kIssuedOff) = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // everything below may read the plan; the combine kernel may be scheduled now (it waits for
    // this grid to finish before it reads anything)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem + kSCol;

    if (warp == kProducerWarp) {
        // ---------------- claims units, loads the block's query rows, streams the tiles chunk by chunk
        if (lane == 0) {
            tma_prefetch_desc(&tmKV2);
            tma_prefetch_desc(&tmKV1);
            tma_prefetch_desc(&tmQ);
            const int units = a.plan_hdr[1] * a.nhb;
            int icount = 0, T = 0;
            // for the drain: loads issued per group (this warp issues the even chunk pairs and the RoPE chunk)
            int issued[kGroups] = {};
            int q_loads = 0;
            bool ok = true;
            while (ok) {
                const int u = atomicAdd(a.claim, 1);
                const int slot = icount % kQD;
                if (icount >= kQD && !wait_or_fail(&bar[I_EMPTY + slot], ((icount / kQD) - 1) & 1, a, err)) break;
                volatile int *q = queue + slot * 8;
                if (u >= units) {
                    q[4] = -1;   // no more work
                    mbar_arrive(&bar[I_FULL + slot]);
                    break;
                }
                const int4 it = a.items[u / a.nhb];
                const int hb = u % a.nhb;
                q[0] = it.x;
                q[1] = hb;
                q[2] = it.y & 0xffff;   // the piece index (the planner keeps the piece count above it)
                q[3] = it.z;
                q[4] = it.w;
                mbar_arrive(&bar[I_FULL + slot]);
                // the previous unit's last S^T product has read the query rows
                if (icount >= 1 && !wait_or_fail(&bar[Q_EMPTY], (icount - 1) & 1, a, err)) break;
                // one box: the block's 64 query rows as 9 chunk tiles of 64 columns
                mbar_arrive_expect_tx(&bar[Q_FULL], kChunks * kQChunkBytes);
                tma_load_4d(smem + kQOff, &tmQ, &bar[Q_FULL], 0, kNh * hb, 0, it.x);
                ++q_loads;
                const int ntl = (it.w - it.z + kTok - 1) / kTok;
                for (int jj = 0; jj < ntl && ok; ++jj, ++T) {
                    const int t0 = it.z + jj * kTok;
                    for (int g = 0; g < kGroups; g += 2) {
                        // the previous tile's PV product has finished with these slots (its O^T block, or
                        // for the last slot the whole product that read P^T there)
                        if (T >= 1 && !wait_or_fail(&bar[g < kGroups - 1 ? EMPTY_PAIR + g : EMPTY_P], (T - 1) & 1,
                                                    a, err)) {
                            ok = false;
                            break;
                        }
                        // TMA costs about the same per instruction up to 32 KB, so the latent chunks come in
                        // pairs (one box of the chunk-outer view); the RoPE chunk alone
                        uint8_t *dst = smem + kSlotOff + 2 * g * kChunkBytes;
                        if (g < kGroups - 1) {
                            mbar_arrive_expect_tx(&bar[CH_FULL + g], 2 * kChunkBytes);
                            tma_load_4d(dst, &tmKV2, &bar[CH_FULL + g], 0, t0, 2 * g, it.x);
                        } else {
                            mbar_arrive_expect_tx(&bar[CH_FULL + g], kChunkBytes);
                            tma_load_3d(dst, &tmKV1, &bar[CH_FULL + g], kMlaLatent, t0, it.x);
                        }
                        ++issued[g];
                    }
                    if (ok) *reinterpret_cast<volatile int *>(smem + kIssuedOff) = T + 1;
                }
                ++icount;
            }
            // leave no copy in flight
            for (int g = 0; g < kGroups; g += 2)
                if (issued[g] >= 1) mbar_wait(&bar[CH_FULL + g], (issued[g] - 1) & 1, a.wait_budget_ns);
            if (q_loads >= 1) mbar_wait(&bar[Q_FULL], (q_loads - 1) & 1, a.wait_budget_ns);
        }
    } else if (warp == kCoProducerWarp) {
        // ---------------- co-producer: the odd latent chunk pairs of every tile, in the producer's order
        if (lane == 0) {
            int icount = 0, T = 0;
            int issued[kGroups] = {};
            bool ok = true;
            while (ok) {
                const int slot = icount % kQD;
                if (!wait_or_fail(&bar[I_FULL + slot], (icount / kQD) & 1, a, err)) break;
                volatile int *q = queue + slot * 8;
                const int b = q[0], t_begin = q[3], t_end = q[4];
                mbar_arrive(&bar[I_EMPTY + slot]);
                if (t_end < 0) break;
                const int ntl = (t_end - t_begin + kTok - 1) / kTok;
                for (int jj = 0; jj < ntl && ok; ++jj, ++T) {
                    const int t0 = t_begin + jj * kTok;
                    for (int g = 1; g < kGroups - 1; g += 2) {
                        if (T >= 1 && !wait_or_fail(&bar[EMPTY_PAIR + g], (T - 1) & 1, a, err)) {
                            ok = false;
                            break;
                        }
                        uint8_t *dst = smem + kSlotOff + 2 * g * kChunkBytes;
                        mbar_arrive_expect_tx(&bar[CH_FULL + g], 2 * kChunkBytes);
                        tma_load_4d(dst, &tmKV2, &bar[CH_FULL + g], 0, t0, 2 * g, b);
                        ++issued[g];
                    }
                }
                ++icount;
            }
            for (int g = 1; g < kGroups - 1; g += 2)
                if (issued[g] >= 1) mbar_wait(&bar[CH_FULL + g], (issued[g] - 1) & 1, a.wait_budget_ns);
        }
    } else if (warp == kPrefetchWarp) {
        // ---------------- L2 prefetcher: tile T of the CTA's stream goes to L2 once the producer has issued
        // tile T - kAhead, so that the producer's loads find their tiles in L2 rather than HBM.  It only
        // reads the unit queue and the producer's count; nothing waits for it.
        if (lane == 0) {
            volatile int *issued = reinterpret_cast<volatile int *>(smem + kIssuedOff);
            int icount = 0, T = 0;
            bool ok = true;
            while (ok) {
                const int slot = icount % kQD;
                if (!wait_or_fail(&bar[I_FULL + slot], (icount / kQD) & 1, a, err)) break;
                volatile int *q = queue + slot * 8;
                const int b = q[0], t_begin = q[3], t_end = q[4];
                mbar_arrive(&bar[I_EMPTY + slot]);
                if (t_end < 0) break;
                const int ntl = (t_end - t_begin + kTok - 1) / kTok;
                for (int jj = 0; jj < ntl; ++jj, ++T) {
                    const uint64_t t0 = global_timer_ns();
                    while (*issued < T - kAhead + 1) {
                        if (*err || global_timer_ns() - t0 > a.wait_budget_ns) {
                            ok = false;   // the producer stopped: nothing more to prefetch
                            break;
                        }
                        __nanosleep(200);
                    }
                    if (!ok) break;
                    const int tt = t_begin + jj * kTok;
                    for (int g = 0; g < kGroups - 1; ++g) tma_prefetch_l2_4d(&tmKV2, 0, tt, 2 * g, b);
                    tma_prefetch_l2_3d(&tmKV1, kMlaLatent, tt, b);
                }
                ++icount;
            }
        }
    } else if (warp == kMmaWarp) {
        // ---------------- MMA issuer: S^T over the 9 chunks, then (once P^T is written) the PV blocks
        if (lane == 0) {
            constexpr uint32_t idesc_s = umma_idesc_bf16(kTok, kNh, 0, 0);
            constexpr uint32_t idesc_o = umma_idesc_bf16(128, kNh, 1, 1);
            const uint32_t slot0 = smem_u32(smem + kSlotOff);
            const uint32_t q0 = smem_u32(smem + kQOff);
            const uint32_t p0 = slot0 + kRopeSlot * kChunkBytes;
            int icount = 0, T = 0;
            bool ok = true;
            while (ok) {
                const int slot = icount % kQD;
                if (!wait_or_fail(&bar[I_FULL + slot], (icount / kQD) & 1, a, err)) break;
                volatile int *q = queue + slot * 8;
                const int t_begin = q[3], t_end = q[4];
                mbar_arrive(&bar[I_EMPTY + slot]);
                if (t_end < 0) break;
                const int ntl = (t_end - t_begin + kTok - 1) / kTok;
                if (!wait_or_fail(&bar[Q_FULL], icount & 1, a, err)) break;
                for (int jj = 0; jj < ntl; ++jj, ++T) {
                    // S^T = KV . Q^T, K = 576 in 36 steps of 16, chunk by chunk as they land
                    for (int c = 0; c < kChunks && ok; ++c) {
                        if ((c & 1) == 0 && !wait_or_fail(&bar[CH_FULL + c / 2], T & 1, a, err)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks) {
                            umma_ss(tS, umma_smem_desc(slot0 + c * kChunkBytes + ks * 32, 16, 1024, 2),
                                    umma_smem_desc(q0 + c * kQChunkBytes + ks * 32, 16, 1024, 2), idesc_s,
                                    (c > 0 || ks > 0) ? 1u : 0u);
                        }
                    }
                    if (!ok) break;
                    umma_commit(&bar[S_FULL]);
                    if (jj == ntl - 1) umma_commit(&bar[Q_EMPTY]);   // the unit's query rows are no longer read
                    // P^T written into the RoPE slot (and the V rows of tokens past the piece zeroed)
                    if (!wait_or_fail(&bar[P_FULL], T & 1, a, err)) break;
                    // the previous unit's epilogue has read O^T
                    if (jj == 0 && icount >= 1 && !wait_or_fail(&bar[O_FREE], (icount - 1) & 1, a, err)) break;
                    tc_fence_after();
#pragma unroll
                    for (int j = 0; j < kLatChunks / 2; ++j) {
                        // A = V^T block j: latent rows 128 j .. 128 j + 127 (chunks 2j, 2j+1, one slot
                        // apart), 16 tokens per step (two 8-row groups 1024 B apart)
                        // B = P^T: 16 tokens per step (two 128-byte core-matrix groups), 8-head blocks 2 KB apart
#pragma unroll
                        for (int ks = 0; ks < kTok / 16; ++ks) {
                            umma_ss(tmem + j * kNh,
                                    umma_smem_desc(slot0 + 2 * j * kChunkBytes + ks * 2048, kChunkBytes, 1024, 2),
                                    umma_smem_desc(p0 + ks * 256, 128, 2048, 0), idesc_o,
                                    (jj > 0 || ks > 0) ? 1u : 0u);
                        }
                        umma_commit(&bar[EMPTY_PAIR + j]);
                    }
                    umma_commit(&bar[EMPTY_P]);
                }
                if (!ok) break;
                umma_commit(&bar[O_FULL]);
                ++icount;
            }
            umma_commit(&bar[DRAIN]);
            mbar_wait(&bar[DRAIN], 0, a.wait_budget_ns);
        }
    } else {
        // ---------------- softmax + epilogue: warpgroup wg takes heads 32 wg .. 32 wg + 31 of the block;
        // thread t owns token t of each tile (lane t of S^T) and latent rows t + 128 j of O^T
        const int wg = warp >> 2;
        const int quarter = warp & 3;
        const int t = quarter * 32 + lane;
        const int hs = wg * kHW;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        float *red = reinterpret_cast<float *>(smem + kRedOff);
        float *lsum = reinterpret_cast<float *>(smem + kLsumOff);
        volatile int *vote = reinterpret_cast<volatile int *>(smem + kVoteOff) + wg * 8;
        uint8_t *pslot = smem + kSlotOff + kRopeSlot * kChunkBytes;
        int icount = 0, T = 0, uses = 0;
        bool ok = true;
        while (ok) {
            const int slot = icount % kQD;
            if (!wait_or_fail(&bar[I_FULL + slot], (icount / kQD) & 1, a, err)) break;
            volatile int *qq = queue + slot * 8;
            const int b = qq[0], hb = qq[1], piece = qq[2], t_begin = qq[3], t_end = qq[4];
            mbar_arrive(&bar[I_EMPTY + slot]);
            if (t_end < 0) break;
            const int ntl = (t_end - t_begin + kTok - 1) / kTok;
            float m_use[kHW], l_part[kHW];
#pragma unroll
            for (int h = 0; h < kHW; ++h) {
                m_use[h] = -INFINITY;
                l_part[h] = 0.f;
            }
            for (int jj = 0; jj < ntl; ++jj, ++T) {
                const int sb = T & 1;
                if (!wait_or_fail(&bar[S_FULL], T & 1, a, err)) { ok = false; break; }
                tc_fence_after();
                uint32_t raw[kHW];
                tmem_ld_hw(tS + lane_off + hs, raw);
                tmem_wait_ld();
                const bool valid = (t_begin + jj * kTok + t) < t_end;
                float x[kHW];
                bool over = false;
#pragma unroll
                for (int h = 0; h < kHW; ++h) {
                    x[h] = valid ? __uint_as_float(raw[h]) * a.qscale : -INFINITY;
                    over |= x[h] > m_use[h] + kMoveThreshold;
                }
                const int wflag = __any_sync(0xffffffffu, over) ? 1 : 0;
                if (lane == 0) vote[sb * 4 + quarter] = wflag;
                if (!group_sync(&bar[GRP + wg], uses, a, err)) { ok = false; break; }
                const bool any_move = (vote[sb * 4 + 0] | vote[sb * 4 + 1] | vote[sb * 4 + 2] | vote[sb * 4 + 3]) != 0;
                float alpha[kHW];
                bool rescale_o = false;
                if (any_move) {
                    // this tile's maximum over its 128 tokens, per head
#pragma unroll
                    for (int h = 0; h < kHW; ++h) {
                        float mx = x[h];
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                        if (lane == 0) red[(sb * 4 + quarter) * kNh + hs + h] = mx;
                    }
                    if (!group_sync(&bar[GRP + wg], uses, a, err)) { ok = false; break; }
#pragma unroll
                    for (int h = 0; h < kHW; ++h) {
                        const float *rr = red + sb * 4 * kNh + hs + h;
                        const float tm = fmaxf(fmaxf(rr[0], rr[kNh]), fmaxf(rr[2 * kNh], rr[3 * kNh]));
                        const float m_new = fmaxf(m_use[h], tm);
                        alpha[h] = 1.f;
                        if (m_new > m_use[h] + kMoveThreshold) {
                            alpha[h] = ex2(m_use[h] - m_new);   // 0 on the unit's first tile
                            m_use[h] = m_new;
                            l_part[h] *= alpha[h];
                            rescale_o = true;
                        }
                    }
                    rescale_o = rescale_o && jj > 0;   // uniform: the warpgroup saw the same maxima
                }
                // P^T into the RoPE slot (S^T has read it), MN-major without swizzle: core matrices of
                // 8 tokens x 8 heads (128 B); the weight sum takes the same bf16-rounded values
                uint8_t *pdst = pslot + (t >> 3) * 128 + (t & 7) * 16;
#pragma unroll
                for (int h8 = 0; h8 < kHW / 8; ++h8) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int h = h8 * 8 + 2 * e;
                        w[e] = pack_bf16x2(ex2(x[h] - m_use[h]), ex2(x[h + 1] - m_use[h + 1]));
                        l_part[h] += bf16_lo(w[e]);
                        l_part[h + 1] += bf16_hi(w[e]);
                    }
                    *reinterpret_cast<uint4 *>(pdst + (hs / 8 + h8) * 2048) = make_uint4(w[0], w[1], w[2], w[3]);
                }
                // The previous tile's PV product is complete here: this tile's RoPE chunk was loaded into
                // the slot that product released, and S^T has read it.
                if (rescale_o) {
#pragma unroll 1
                    for (int j = 0; j < kLatChunks / 2; ++j) {
                        uint32_t o[kHW];
                        tmem_ld_hw(tmem + j * kNh + lane_off + hs, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int h = 0; h < kHW; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
                        tmem_st_hw(tmem + j * kNh + lane_off + hs, o);
                    }
                    tmem_wait_st();
                }
                if (!valid) {
                    // Rows past the piece may hold anything (NaN included) and the tensor cores would
                    // form 0 * NaN: the token's latent row is zeroed once it has landed (each warpgroup
                    // zeroes its share of the eight chunks)
                    constexpr int kZ = kLatChunks / kNWG;
#pragma unroll
                    for (int c = 0; c < kZ; ++c) {
                        const int ch = wg * kZ + c;
                        if (!wait_or_fail(&bar[CH_FULL + ch / 2], T & 1, a, err)) { ok = false; break; }
                        uint4 *row = reinterpret_cast<uint4 *>(smem + kSlotOff + ch * kChunkBytes + t * 128);
#pragma unroll
                        for (int i = 0; i < 8; ++i) row[i] = make_uint4(0u, 0u, 0u, 0u);
                    }
                    if (!ok) break;
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&bar[P_FULL]);
            }
            if (!ok) break;

            // ---------------- epilogue of the unit: weight sums over the 128 tokens, then O^T
#pragma unroll
            for (int h = 0; h < kHW; ++h) {
                float v = l_part[h];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0) lsum[quarter * kNh + hs + h] = v;
            }
            if (!group_sync(&bar[GRP + wg], uses, a, err)) break;
            if (!wait_or_fail(&bar[O_FULL], icount & 1, a, err)) break;
            tc_fence_after();
            const bool whole = a.nsplit_b[b] == 1;
            const int h0 = hb * kNh + hs;
#pragma unroll 1
            for (int j = 0; j < kLatChunks / 2; ++j) {
                uint32_t o[kHW];
                tmem_ld_hw(tmem + j * kNh + lane_off + hs, o);
                tmem_wait_ld();
                const int d = j * 128 + t;
#pragma unroll
                for (int h = 0; h < kHW; ++h) {
                    const int hg = h0 + h;
                    if (hg >= a.Hq) continue;
                    const float L = lsum[hs + h] + lsum[kNh + hs + h] + lsum[2 * kNh + hs + h] + lsum[3 * kNh + hs + h];
                    const float O = __uint_as_float(o[h]);
                    const size_t row = (size_t)b * a.Hq + hg;
                    if (whole) {
                        // a zero sum only for an empty history (output 0); a NaN sum (a NaN in the cache)
                        // stays NaN
                        a.out[row * kMlaLatent + d] = __float2bfloat16_rn(L != 0.f ? O / L : 0.f);
                    } else {
                        const size_t prow = row * a.nsplit + piece;
                        a.part_o[prow * kMlaLatent + d] = O;
                        if (d == 0) {
                            a.part_ml[prow * 2 + 0] = m_use[h];
                            a.part_ml[prow * 2 + 1] = L;
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&bar[O_FREE]);
            ++icount;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// One CTA per (head, sequence) of a split history, four latent coordinates per thread: the pieces'
// partials merged with weights 2^(m_s - M), M their largest maximum.  Launched as a programmatic
// dependent of the decode kernel; histories of one piece were written out by it.
__global__ void __launch_bounds__(kMlaLatent / 4) mla_combine_planned_kernel(const MlaTcArgs a)
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int h = blockIdx.x, b = blockIdx.y;
    const int nv = min(a.nsplit_b[b], a.nsplit);
    if (nv <= 1) return;
    const int d = threadIdx.x * 4;
    const size_t row = (size_t)b * a.Hq + h;
    const float *ml = a.part_ml + row * a.nsplit * 2;
    float M = -INFINITY;
    for (int s = 0; s < nv; ++s) M = fmaxf(M, ml[2 * s]);
    float L = 0.f, O[4] = {0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < nv; ++s) {
        const float m = ml[2 * s];
        const float w = (m == -INFINITY) ? 0.f : ex2(m - M);
        L += ml[2 * s + 1] * w;
        const float4 p = *reinterpret_cast<const float4 *>(a.part_o + (row * a.nsplit + s) * kMlaLatent + d);
        O[0] += p.x * w;
        O[1] += p.y * w;
        O[2] += p.z * w;
        O[3] += p.w * w;
    }
    // a NaN sum (a NaN in the cache) stays NaN
    uint2 packed;
    packed.x = pack_bf16x2(O[0] / L, O[1] / L);
    packed.y = pack_bf16x2(O[2] / L, O[3] / L);
    *reinterpret_cast<uint2 *>(a.out + row * kMlaLatent + d) = packed;
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

MlaTcPlan mla_tc_plan_host(int B, int Hq, int Tmax, size_t ws_budget)
{
    MlaTcPlan p{};
    const long long tiles = (Tmax + kTok - 1) / kTok;
    // at most 64 pieces per sequence, fewer when their partials would not fit the budget
    const size_t per_piece = (size_t)B * Hq * (kMlaLatent + 2) * 4 + (size_t)B * 16;
    long long cap = tiles < 64 ? tiles : 64;
    const long long fit = (long long)(ws_budget / per_piece);
    if (fit < cap) cap = fit < 1 ? 1 : fit;
    p.nsplit = (int)cap;
    p.nhb = (Hq + kNh - 1) / kNh;
    size_t off = 0;
    p.off_hdr = off;
    off += 256;
    p.off_nsb = off;
    off += round256((size_t)B * 4);   // pieces per sequence
    p.off_items = off;
    off += round256((size_t)B * p.nsplit * 16);
    p.off_po = off;
    off += round256((size_t)B * Hq * p.nsplit * kMlaLatent * 4);
    p.off_pml = off;
    off += round256((size_t)B * Hq * p.nsplit * 2 * 4);
    p.ws_bytes = off;
    return p;
}

cudaError_t launch_mla_decode_tc(const CUtensorMap &tmKV2, const CUtensorMap &tmKV1, const CUtensorMap &tmQ,
                                 const void *q,
                                 const int32_t *seqlens, int B, int Hq, int Tmax, float scale, void *out, void *ws,
                                 const MlaTcPlan &p, int num_sms, int *status, unsigned long long wait_budget_ns,
                                 cudaStream_t stream, int *launches, cudaEvent_t before, cudaEvent_t after)
{
    (void)q;
    uint8_t *w = static_cast<uint8_t *>(ws);
    // the planner: pieces from the real lengths, about two rounds of (piece, head block) units per CTA
    DecodeArgs pa{};
    pa.seqlens = seqlens;
    pa.out = static_cast<__nv_bfloat16 *>(out);
    pa.status = status;
    pa.B = B;
    pa.Hq = Hq;
    pa.Hkv = p.nhb;
    pa.Tmax = Tmax;
    pa.group = kNh;
    pa.nsplit = p.nsplit;
    pa.plan_hdr = reinterpret_cast<int *>(w + p.off_hdr);
    pa.nsplit_b = reinterpret_cast<int *>(w + p.off_nsb);
    pa.items = reinterpret_cast<int4 *>(w + p.off_items);
    pa.num_ctas = num_sms;
    pa.out_row = kMlaLatent;
    // one round of long pieces per CTA, each history's remainder cut into four (a sweep over 1-6 rounds
    // and 1-4 tail pieces at the DeepSeek-V3 shape: 190 -> 180 us against two rounds of whole pieces)
    pa.plan_rounds = 1;
    pa.tail_split = 4;
    cudaError_t e = launch_decode_plan(pa, stream);
    if (e != cudaSuccess) return e;
    ++*launches;

    MlaTcArgs a{};
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.part_o = reinterpret_cast<float *>(w + p.off_po);
    a.part_ml = reinterpret_cast<float *>(w + p.off_pml);
    a.status = status;
    a.plan_hdr = pa.plan_hdr;
    a.claim = pa.plan_hdr;
    a.nsplit_b = pa.nsplit_b;
    a.items = pa.items;
    a.B = B;
    a.Hq = Hq;
    a.nsplit = p.nsplit;
    a.nhb = p.nhb;
    a.qscale = scale * 1.4426950408889634f;   // log2(e): the softmax runs in base 2
    a.wait_budget_ns = wait_budget_ns;

    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
        if ((e = cudaFuncSetAttribute(mla_decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      kSmemBytes)) != cudaSuccess)
            return e;
        attr_done[dev] = true;
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(num_sms);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (before) cudaEventRecord(before, stream);
    if ((e = cudaLaunchKernelEx(&cfg, mla_decode_tc_kernel, tmKV2, tmKV1, tmQ, a)) != cudaSuccess) return e;
    if (after) cudaEventRecord(after, stream);
    ++*launches;

    cudaLaunchConfig_t cc = {};
    cc.gridDim = dim3(Hq, B);
    cc.blockDim = dim3(kMlaLatent / 4);
    cc.stream = stream;
    cc.attrs = attr;
    cc.numAttrs = 1;
    if ((e = cudaLaunchKernelEx(&cc, mla_combine_planned_kernel, a)) != cudaSuccess) return e;
    ++*launches;
    return cudaSuccess;
}

}  // namespace gqa
