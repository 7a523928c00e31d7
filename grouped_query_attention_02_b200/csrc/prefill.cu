// prefill.cu -- causal GQA prefill on the tcgen05 tensor cores.
//
// One CTA computes one 128-row query tile of one (sequence, query head).  The
// query head h reads KV head h / g ("grouped-query and multi-query attention",
// study.greatitself.com: consecutive groups); K/V tiles are fetched by TMA and
// the g query heads of a group run as neighbouring CTAs so that a tile read
// from HBM serves the whole group out of L2.  The causal mask of
// anrans.github.io attention-variants ("Kernels do not need to copy the KV
// heads": lower triangle, diagonal included) is applied inside the diagonal
// tile only; tiles above the diagonal are never visited.
//
// Warp roles (192 threads):
//   warp 0      TMA producer: the Q tile once, then K_j / V_j into a two-stage ring
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer:
//               S_j = Q K_j^T into one of two TMEM buffers, O += P_j V_j into TMEM
//   warps 2..5  softmax: one query row per thread, read straight from TMEM
//               (warp w may touch TMEM lanes 32*(w%4) .. +31), online softmax in
//               base 2 with fp32 state, P_j rounded to bf16 into shared memory,
//               then the epilogue O / l -> bf16 -> global.
//
// The running maximum is only moved when a row's new maximum exceeds it by
// more than 8 (in log2 units); otherwise the weights are taken against the old
// maximum (they stay below 2^8, exact in fp32) and the O accumulator in TMEM
// needs no rescale.  The final division by l uses the same maximum, so the
// result is the same softmax.
//
// Shared memory (1024-byte aligned, 128-byte swizzle everywhere):
//   Q [2 halves][128 rows][128 B]  32 KB
//   K [2 stages][2 halves][128][128 B]  64 KB,  V likewise 64 KB
//   P [2 halves][128 rows][128 B]  32 KB
#include "internal.h"
#include "ptx.cuh"

namespace gqa {

namespace {

constexpr int kD = kHeadDim;
constexpr int kBM = 128;                   // query rows per CTA
constexpr int kBN = 128;                   // keys per KV tile
constexpr int kTileBytes = kBM * kD * 2;   // 32 KB: one 128 x 128 bf16 tile
constexpr int kHalfTile = kTileBytes / 2;  // one 64-column half
constexpr int kThreads = 192;
constexpr int kSoftmaxThreads = 128;
constexpr uint32_t kTmemCols = 512;        // S0, S1, O (128 columns each), rounded to a power of two
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct Smem {
    static constexpr int q = 0;
    static constexpr int k = q + kTileBytes;
    static constexpr int v = k + 2 * kTileBytes;
    static constexpr int p = v + 2 * kTileBytes;
    static constexpr int bars = p + kTileBytes;
    // barriers: q_full, k_full[2], v_full[2], kv_empty[2], s_full[2], s_free[2], p_full, p_free, o_full, drain
    static constexpr int nbars = 15;
    static constexpr int tmem_slot = bars + nbars * 8;
    static constexpr int err = tmem_slot + 8;
    static constexpr int bytes = err + 8;
};

enum Bar {
    Q_FULL = 0, K_FULL = 1, V_FULL = 3, KV_EMPTY = 5, S_FULL = 7, S_FREE = 9,
    P_FULL = 11, P_FREE = 12, O_FULL = 13, DRAIN = 14
};

__device__ __forceinline__ void record_status(int *status, int code)
{
    if (status) atomicCAS(status, 0, code);
}

// bounded wait that also gives up as soon as another role has reported an error
__device__ __forceinline__ bool wait_or_fail(uint64_t *bar, uint32_t parity, const PrefillArgs &a,
                                             volatile int *err)
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

// K-major operand with 128-byte swizzle: rows of 128 B, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t saddr) { return umma_smem_desc(saddr, 16, 1024, 2); }
// MN-major operand with 128-byte swizzle: 64-element column blocks `lbo` bytes apart, 8-row K groups 1024 B apart.
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t saddr, uint32_t lbo)
{
    return umma_smem_desc(saddr, lbo, 1024, 2);
}

// max of three floats in one instruction (PTX max.f32 with three sources, sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__global__ void __launch_bounds__(kThreads, 1)
prefill_causal_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const PrefillArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + Smem::bars);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Smem::tmem_slot);
    volatile int *err = reinterpret_cast<volatile int *>(smem + Smem::err);

    // heaviest query tiles first over the whole grid; a group's heads are neighbours
    const int nqt = (a.S + kBM - 1) / kBM;
    const int bh_count = a.B * a.Hq;
    const int id = blockIdx.x;
    const int qt = nqt - 1 - id / bh_count;
    const int bh = id % bh_count;
    const int b = bh / a.Hq;
    const int h = bh % a.Hq;
    const int kvh = h / a.group;
    const int q0 = qt * kBM;
    const int ntiles = qt + 1;             // KV tiles 0..qt (causal)

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&bar[Q_FULL], 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar[K_FULL + s], 1);
            mbar_init(&bar[V_FULL + s], 1);
            mbar_init(&bar[KV_EMPTY + s], 1);
            mbar_init(&bar[S_FULL + s], 1);
            mbar_init(&bar[S_FREE + s], kSoftmaxThreads);
        }
        mbar_init(&bar[P_FULL], kSoftmaxThreads);
        mbar_init(&bar[P_FREE], 1);
        mbar_init(&bar[O_FULL], 1);
        mbar_init(&bar[DRAIN], 1);
        *err = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS[2] = {tmem, tmem + 128};
    const uint32_t tO = tmem + 256;

    if (warp == 0) {
        // ---------------- TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            mbar_arrive_expect_tx(&bar[Q_FULL], kTileBytes);
            tma_load_4d(smem + Smem::q, &tmQ, &bar[Q_FULL], 0, h, q0, b);
            tma_load_4d(smem + Smem::q + kHalfTile, &tmQ, &bar[Q_FULL], 64, h, q0, b);
            int issued = 0;
            for (int j = 0; j < ntiles; ++j) {
                const int s = j & 1;
                if (j >= 2 && !wait_or_fail(&bar[KV_EMPTY + s], ((j >> 1) - 1) & 1, a, err)) break;
                uint8_t *ks = smem + Smem::k + s * kTileBytes;
                uint8_t *vs = smem + Smem::v + s * kTileBytes;
                mbar_arrive_expect_tx(&bar[K_FULL + s], kTileBytes);
                tma_load_4d(ks, &tmK, &bar[K_FULL + s], 0, kvh, j * kBN, b);
                tma_load_4d(ks + kHalfTile, &tmK, &bar[K_FULL + s], 64, kvh, j * kBN, b);
                mbar_arrive_expect_tx(&bar[V_FULL + s], kTileBytes);
                tma_load_4d(vs, &tmV, &bar[V_FULL + s], 0, kvh, j * kBN, b);
                tma_load_4d(vs + kHalfTile, &tmV, &bar[V_FULL + s], 64, kvh, j * kBN, b);
                ++issued;
            }
            // leave no copy in flight: the last loads of each stage and the Q tile must have landed
            for (int j = issued - 1; j >= 0 && j >= issued - 2; --j) {
                const uint32_t ph = (j >> 1) & 1;
                mbar_wait(&bar[K_FULL + (j & 1)], ph, a.wait_budget_ns);
                mbar_wait(&bar[V_FULL + (j & 1)], ph, a.wait_budget_ns);
            }
            mbar_wait(&bar[Q_FULL], 0, a.wait_budget_ns);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (one thread)
        if (lane == 0) {
            const uint32_t idesc_s = umma_idesc_bf16(kBM, kBN, 0, 0);   // Q (K-major) x K (K-major)
            const uint32_t idesc_o = umma_idesc_bf16(kBM, kD, 0, 1);    // P (K-major) x V (MN-major)
            const uint32_t q_addr = smem_u32(smem + Smem::q);
            const uint32_t p_addr = smem_u32(smem + Smem::p);
            bool ok = wait_or_fail(&bar[Q_FULL], 0, a, err);
            int pv_done = 0;
            for (int j = 0; ok && j <= ntiles; ++j) {
                if (j < ntiles) {
                    const int s = j & 1;
                    if (!wait_or_fail(&bar[K_FULL + s], (j >> 1) & 1, a, err)) { ok = false; break; }
                    if (j >= 2 && !wait_or_fail(&bar[S_FREE + s], ((j >> 1) - 1) & 1, a, err)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t k_addr = smem_u32(smem + Smem::k + s * kTileBytes);
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks) {
                        const uint32_t off = (ks >> 2) * kHalfTile + (ks & 3) * 32;
                        umma_ss(tS[s], desc_kmajor(q_addr + off), desc_kmajor(k_addr + off), idesc_s,
                                     ks > 0 ? 1u : 0u);
                    }
                    umma_commit(&bar[S_FULL + s]);
                }
                if (j >= 1) {
                    const int jp = j - 1;      // PV of the previous tile
                    const int s = jp & 1;
                    if (!wait_or_fail(&bar[P_FULL], jp & 1, a, err)) { ok = false; break; }
                    if (!wait_or_fail(&bar[V_FULL + s], (jp >> 1) & 1, a, err)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t v_addr = smem_u32(smem + Smem::v + s * kTileBytes);
#pragma unroll
                    for (int ks = 0; ks < kBN / 16; ++ks) {
                        const uint32_t poff = (ks >> 2) * kHalfTile + (ks & 3) * 32;
                        umma_ss(tO, desc_kmajor(p_addr + poff), desc_mnmajor(v_addr + ks * 2048, kHalfTile),
                                     idesc_o, (jp > 0 || ks > 0) ? 1u : 0u);
                    }
                    umma_commit(&bar[P_FREE]);
                    umma_commit(&bar[KV_EMPTY + s]);
                    ++pv_done;
                }
            }
            if (ok && pv_done == ntiles) umma_commit(&bar[O_FULL]);
            // no MMA may still run when TMEM is released
            umma_commit(&bar[DRAIN]);
            mbar_wait(&bar[DRAIN], 0, a.wait_budget_ns);
        }
    } else {
        // ---------------- softmax warps: thread owns query row r of the tile
        const int quarter = warp & 3;                 // TMEM lane quarter this warp may access
        const int r = quarter * 32 + lane;            // row within the tile
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int qrow = q0 + r;
        uint8_t *prow = smem + Smem::p + r * 128;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int j = 0; j < ntiles; ++j) {
            const int s = j & 1;
            if (!wait_or_fail(&bar[S_FULL + s], (j >> 1) & 1, a, err)) { ok = false; break; }
            tc_fence_after();
            uint32_t sr[128];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tS[s] + lane_off + c * 32, sr + c * 32);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&bar[S_FREE + s]);

            // raw scores; the diagonal tile hides keys after the row.  Eight independent partial maxima
            // keep the reduction off a 128-long dependency chain.
            const bool diag = (j == qt);
            float pm[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) pm[i] = -INFINITY;
#pragma unroll
            for (int c = 0; c < 128; ++c) {
                if (diag && c > r) sr[c] = __float_as_uint(-INFINITY);
                pm[c & 7] = fmaxf(pm[c & 7], __uint_as_float(sr[c]));
            }
            const float mraw = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                                     fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
            // in log2 units: qscale = log2(e)/sqrt(d) > 0, so max(raw)*qscale is the scaled maximum
            const float m_new = fmaxf(m_run, mraw * a.qscale);
            const bool move = (m_new > m_run + kRescaleThreshold);
            const float m_use = move ? m_new : m_run;
            const float alpha = move ? ex2(m_run - m_new) : 1.f;   // ex2(-inf) = 0 on the first tile
            // p = 2^(raw*qscale - m_use): one packed FMA per two elements, then the exp unit
            const float2 sc2 = make_float2(a.qscale, a.qscale);
            const float2 nm2 = make_float2(-m_use, -m_use);
            float2 ps[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                            make_float2(0.f, 0.f)};
            float x[128];
#pragma unroll
            for (int c = 0; c < 128; c += 2) {
                const float2 e = __ffma2_rn(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sc2, nm2);
                const float2 pe = make_float2(ex2(e.x), ex2(e.y));
                x[c] = pe.x;
                x[c + 1] = pe.y;
                ps[(c >> 1) & 3] = __fadd2_rn(ps[(c >> 1) & 3], pe);
            }
            const float rs = (ps[0].x + ps[0].y) + (ps[1].x + ps[1].y) + (ps[2].x + ps[2].y) + (ps[3].x + ps[3].y);
            m_run = m_use;
            l_run = l_run * alpha + rs;

            if (j >= 1) {
                // previous PV done: P buffer free, O stable
                if (!wait_or_fail(&bar[P_FREE], (j - 1) & 1, a, err)) { ok = false; break; }
                tc_fence_after();
                if (__any_sync(0xffffffffu, move)) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t orow[32];
                        tmem_ld32(tO + lane_off + c * 32, orow);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) orow[i] = __float_as_uint(__uint_as_float(orow[i]) * alpha);
                        tmem_st32(tO + lane_off + c * 32, orow);
                    }
                    tmem_wait_st();
                }
            }
            // P row -> bf16, K-major with the 128-byte swizzle: 16-byte chunk c of half hh at chunk c ^ (r & 7)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const int e = hh * 64 + c * 8;
                    uint4 w;
                    w.x = pack_bf16x2(x[e + 0], x[e + 1]);
                    w.y = pack_bf16x2(x[e + 2], x[e + 3]);
                    w.z = pack_bf16x2(x[e + 4], x[e + 5]);
                    w.w = pack_bf16x2(x[e + 6], x[e + 7]);
                    *reinterpret_cast<uint4 *>(prow + hh * kHalfTile + ((c ^ (r & 7)) << 4)) = w;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bar[P_FULL]);
        }
        if (ok && wait_or_fail(&bar[O_FULL], 0, a, err)) {
            tc_fence_after();
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            // log-sum-exp of the row's scaled scores, natural log: (m + log2 l) ln 2
            if (a.lse && qrow < a.S)
                a.lse[((size_t)b * a.Hq + h) * a.S + qrow] = (m_run + __log2f(l_run)) * 0.6931471805599453f;
            __nv_bfloat16 *orow_g = a.out + (((size_t)b * a.S + qrow) * a.Hq + h) * kD;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t orow[32];
                tmem_ld32(tO + lane_off + c * 32, orow);
                tmem_wait_ld();
                if (qrow < a.S) {
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(orow[i + 0]) * inv, __uint_as_float(orow[i + 1]) * inv);
                        w.y = pack_bf16x2(__uint_as_float(orow[i + 2]) * inv, __uint_as_float(orow[i + 3]) * inv);
                        w.z = pack_bf16x2(__uint_as_float(orow[i + 4]) * inv, __uint_as_float(orow[i + 5]) * inv);
                        w.w = pack_bf16x2(__uint_as_float(orow[i + 6]) * inv, __uint_as_float(orow[i + 7]) * inv);
                        *reinterpret_cast<uint4 *>(orow_g + c * 32 + i) = w;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}


// ----------------------------------------------------------------------------
// Paired-head variant for even group sizes.  One CTA computes the same
// 128-row query tile of two query heads of one group (h, h+1): they read the
// same KV head, so every K/V tile in shared memory serves both, and they have
// the same causal shape.  Two softmax warpgroups (one per head) alternate on
// the tensor core: while one works through its softmax, the MMAs of the other
// run.  Each warpgroup's P goes back into tensor memory over its own S (bf16,
// two per 32-bit column) and the PV product reads it from there, so both Q
// tiles and a two-stage K/V ring fit in shared memory.
//
// Warps: 0..3 softmax of head h, 4..7 softmax of head h+1 (TMEM lane quarter =
// warp % 4), 8 TMA producer, 9 TMEM allocator + MMA issuer.
// TMEM columns: S_A 0..127 (P_A over 0..63), S_B 128..255, O_A 256..383, O_B 384..511.
constexpr int kPairThreads = 320;

struct PairSmem {
    static constexpr int q = 0;                          // Q_A then Q_B, 32 KB each
    static constexpr int kv = 2 * kTileBytes;            // stage s: K at kv + s*64K, V at +32K
    static constexpr int bars = kv + 4 * kTileBytes;
    // q_full, k_full[2], v_full[2], kv_empty[2], s_full[2], p_full[2], o_full, drain
    static constexpr int nbars = 13;
    static constexpr int tmem_slot = bars + nbars * 8;
    static constexpr int err = tmem_slot + 8;
    static constexpr int bytes = err + 8;
};

enum PairBar { PQ_FULL = 0, PK_FULL = 1, PV_FULL = 3, PKV_EMPTY = 5, PS_FULL = 7, PP_FULL = 9, PO_FULL = 11,
               PDRAIN = 12 };

__global__ void __launch_bounds__(kPairThreads, 1)
prefill_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const PrefillArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + PairSmem::bars);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + PairSmem::tmem_slot);
    volatile int *err = reinterpret_cast<volatile int *>(smem + PairSmem::err);

    // heaviest query tiles first; the pairs of one group are neighbours
    const int nqt = (a.S + kBM - 1) / kBM;
    const int pairs = a.Hq / 2;
    const int per_qt = a.B * pairs;
    const int id = blockIdx.x;
    const int qt = nqt - 1 - id / per_qt;
    const int rem = id % per_qt;
    const int b = rem / pairs;
    const int hA = 2 * (rem % pairs);
    const int kvh = hA / a.group;
    const int q0 = qt * kBM;
    const int ntiles = qt + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&bar[PQ_FULL], 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar[PK_FULL + s], 1);
            mbar_init(&bar[PV_FULL + s], 1);
            mbar_init(&bar[PKV_EMPTY + s], 1);
            mbar_init(&bar[PS_FULL + s], 1);
            mbar_init(&bar[PP_FULL + s], kSoftmaxThreads);
        }
        mbar_init(&bar[PO_FULL], 1);
        mbar_init(&bar[PDRAIN], 1);
        *err = 0;
        fence_barrier_init();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 8) {
        // ---------------- TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            mbar_arrive_expect_tx(&bar[PQ_FULL], 2 * kTileBytes);
            for (int w = 0; w < 2; ++w) {
                uint8_t *qs = smem + PairSmem::q + w * kTileBytes;
                tma_load_4d(qs, &tmQ, &bar[PQ_FULL], 0, hA + w, q0, b);
                tma_load_4d(qs + kHalfTile, &tmQ, &bar[PQ_FULL], 64, hA + w, q0, b);
            }
            int issued = 0;
            for (int j = 0; j < ntiles; ++j) {
                const int s = j & 1;
                if (j >= 2 && !wait_or_fail(&bar[PKV_EMPTY + s], ((j >> 1) - 1) & 1, a, err)) break;
                uint8_t *ks = smem + PairSmem::kv + s * 2 * kTileBytes;
                uint8_t *vs = ks + kTileBytes;
                mbar_arrive_expect_tx(&bar[PK_FULL + s], kTileBytes);
                tma_load_4d(ks, &tmK, &bar[PK_FULL + s], 0, kvh, j * kBN, b);
                tma_load_4d(ks + kHalfTile, &tmK, &bar[PK_FULL + s], 64, kvh, j * kBN, b);
                mbar_arrive_expect_tx(&bar[PV_FULL + s], kTileBytes);
                tma_load_4d(vs, &tmV, &bar[PV_FULL + s], 0, kvh, j * kBN, b);
                tma_load_4d(vs + kHalfTile, &tmV, &bar[PV_FULL + s], 64, kvh, j * kBN, b);
                ++issued;
            }
            for (int j = issued - 1; j >= 0 && j >= issued - 2; --j) {
                const uint32_t ph = (j >> 1) & 1;
                mbar_wait(&bar[PK_FULL + (j & 1)], ph, a.wait_budget_ns);
                mbar_wait(&bar[PV_FULL + (j & 1)], ph, a.wait_budget_ns);
            }
            mbar_wait(&bar[PQ_FULL], 0, a.wait_budget_ns);
        }
    } else if (warp == 9) {
        // ---------------- MMA issuer: S_A(0) S_B(0) | PV_A(j) S_A(j+1) PV_B(j) S_B(j+1) | ...
        if (lane == 0) {
            const uint32_t idesc_s = umma_idesc_bf16(kBM, kBN, 0, 0);   // Q (K-major) x K (K-major)
            const uint32_t idesc_o = umma_idesc_bf16(kBM, kD, 0, 1);    // P (TMEM) x V (MN-major)
            const uint32_t q_addr = smem_u32(smem + PairSmem::q);
            bool ok = wait_or_fail(&bar[PQ_FULL], 0, a, err) && wait_or_fail(&bar[PK_FULL], 0, a, err);
            auto issue_s = [&](int w, int j) {
                const uint32_t k_addr = smem_u32(smem + PairSmem::kv + (j & 1) * 2 * kTileBytes);
                const uint32_t qa = q_addr + w * kTileBytes;
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * kHalfTile + (ks & 3) * 32;
                    umma_ss(tmem + w * 128, desc_kmajor(qa + off), desc_kmajor(k_addr + off), idesc_s,
                                 ks > 0 ? 1u : 0u);
                }
                umma_commit(&bar[PS_FULL + w]);
            };
            if (ok) {
                tc_fence_after();
                issue_s(0, 0);
                issue_s(1, 0);
            }
            int pv_done = 0;
            for (int j = 0; ok && j < ntiles; ++j) {
                const int s = j & 1;
                const uint32_t v_addr = smem_u32(smem + PairSmem::kv + s * 2 * kTileBytes + kTileBytes);
                for (int w = 0; w < 2; ++w) {
                    if (!wait_or_fail(&bar[PP_FULL + w], j & 1, a, err)) { ok = false; break; }
                    if (w == 0 && !wait_or_fail(&bar[PV_FULL + s], (j >> 1) & 1, a, err)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < kBN / 16; ++ks) {
                        // A = P: 16 keys = 8 columns of packed bf16 pairs; B = V rows ks*16 .. +16
                        umma_ts(tmem + 256 + w * 128, tmem + w * 128 + ks * 8,
                                     desc_mnmajor(v_addr + ks * 2048, kHalfTile), idesc_o,
                                     (j > 0 || ks > 0) ? 1u : 0u);
                    }
                    if (w == 1) {
                        umma_commit(&bar[PKV_EMPTY + s]);
                        ++pv_done;
                    }
                    if (j + 1 < ntiles) {
                        if (w == 0 && !wait_or_fail(&bar[PK_FULL + ((j + 1) & 1)], ((j + 1) >> 1) & 1, a, err)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        issue_s(w, j + 1);
                    }
                }
            }
            if (ok && pv_done == ntiles) umma_commit(&bar[PO_FULL]);
            umma_commit(&bar[PDRAIN]);
            mbar_wait(&bar[PDRAIN], 0, a.wait_budget_ns);
        }
    } else {
        // ---------------- softmax warpgroup w: head hA + w, thread owns query row r
        const int w = warp >> 2;
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t tS = tmem + w * 128 + lane_off;
        const uint32_t tO = tmem + 256 + w * 128 + lane_off;
        const int qrow = q0 + r;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int j = 0; j < ntiles; ++j) {
            if (!wait_or_fail(&bar[PS_FULL + w], j & 1, a, err)) { ok = false; break; }
            tc_fence_after();
            const bool diag = (j == qt);
            // pass 1: the row maximum of the raw scores (keys after the row hidden on the diagonal);
            // two 32-column loads per wait, three-input max, four independent partial maxima
            float pm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int c2 = 0; c2 < 4; c2 += 2) {
                uint32_t sr[64];
                tmem_ld32(tS + c2 * 32, sr);
                tmem_ld32(tS + c2 * 32 + 32, sr + 32);
                tmem_wait_ld();
                if (diag) {
#pragma unroll
                    for (int i = 0; i < 64; ++i)
                        if (c2 * 32 + i > r) sr[i] = __float_as_uint(-INFINITY);
                }
#pragma unroll
                for (int i = 0; i < 64; i += 8) {
                    pm[0] = fmax3(pm[0], __uint_as_float(sr[i + 0]), __uint_as_float(sr[i + 1]));
                    pm[1] = fmax3(pm[1], __uint_as_float(sr[i + 2]), __uint_as_float(sr[i + 3]));
                    pm[2] = fmax3(pm[2], __uint_as_float(sr[i + 4]), __uint_as_float(sr[i + 5]));
                    pm[3] = fmax3(pm[3], __uint_as_float(sr[i + 6]), __uint_as_float(sr[i + 7]));
                }
            }
            const float mraw = fmaxf(fmax3(pm[0], pm[1], pm[2]), pm[3]);
            const float m_new = fmaxf(m_run, mraw * a.qscale);
            const bool move = (m_new > m_run + kRescaleThreshold);
            const float m_use = move ? m_new : m_run;
            const float alpha = move ? ex2(m_run - m_new) : 1.f;
            // O holds tiles < j (the S_FULL commit covers the previous PV): rescale when the max moved
            if (j > 0 && __any_sync(0xffffffffu, move)) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t orow[32];
                    tmem_ld32(tO + c * 32, orow);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) orow[i] = __float_as_uint(__uint_as_float(orow[i]) * alpha);
                    tmem_st32(tO + c * 32, orow);
                }
            }
            // pass 2: p = 2^(raw*qscale - m_use), summed, packed to bf16 pairs over S columns 0..63
            const float2 sc2 = make_float2(a.qscale, a.qscale);
            const float2 nm2 = make_float2(-m_use, -m_use);
            float2 ps[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                            make_float2(0.f, 0.f)};
#pragma unroll
            for (int c2 = 0; c2 < 4; c2 += 2) {
                uint32_t sr[64];
                tmem_ld32(tS + c2 * 32, sr);
                tmem_ld32(tS + c2 * 32 + 32, sr + 32);
                tmem_wait_ld();
                if (diag) {
#pragma unroll
                    for (int i = 0; i < 64; ++i)
                        if (c2 * 32 + i > r) sr[i] = __float_as_uint(-INFINITY);
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        const float2 e = __ffma2_rn(
                            make_float2(__uint_as_float(sr[h * 32 + i]), __uint_as_float(sr[h * 32 + i + 1])), sc2, nm2);
                        const float2 pe = make_float2(ex2(e.x), ex2(e.y));
                        ps[(i >> 1) & 3] = __fadd2_rn(ps[(i >> 1) & 3], pe);
                        pk[i >> 1] = pack_bf16x2(pe.x, pe.y);
                    }
                    tmem_st16(tS + (c2 + h) * 16, pk);
                }
            }
            tmem_wait_st();
            const float rs = (ps[0].x + ps[0].y) + (ps[1].x + ps[1].y) + (ps[2].x + ps[2].y) + (ps[3].x + ps[3].y);
            m_run = m_use;
            l_run = l_run * alpha + rs;
            tc_fence_before();
            mbar_arrive(&bar[PP_FULL + w]);
        }
        if (ok && wait_or_fail(&bar[PO_FULL], 0, a, err)) {
            tc_fence_after();
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            // log-sum-exp of the row's scaled scores, natural log: (m + log2 l) ln 2
            if (a.lse && qrow < a.S)
                a.lse[((size_t)b * a.Hq + hA + w) * a.S + qrow] = (m_run + __log2f(l_run)) * 0.6931471805599453f;
            __nv_bfloat16 *orow_g = a.out + (((size_t)b * a.S + qrow) * a.Hq + hA + w) * kD;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t orow[32];
                tmem_ld32(tO + c * 32, orow);
                tmem_wait_ld();
                if (qrow < a.S) {
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        uint4 v;
                        v.x = pack_bf16x2(__uint_as_float(orow[i + 0]) * inv, __uint_as_float(orow[i + 1]) * inv);
                        v.y = pack_bf16x2(__uint_as_float(orow[i + 2]) * inv, __uint_as_float(orow[i + 3]) * inv);
                        v.z = pack_bf16x2(__uint_as_float(orow[i + 4]) * inv, __uint_as_float(orow[i + 5]) * inv);
                        v.w = pack_bf16x2(__uint_as_float(orow[i + 6]) * inv, __uint_as_float(orow[i + 7]) * inv);
                        *reinterpret_cast<uint4 *>(orow_g + c * 32 + i) = v;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

cudaError_t launch_prefill(const CUtensorMap &tmQ, const CUtensorMap &tmK, const CUtensorMap &tmV,
                           const PrefillArgs &a, cudaStream_t stream)
{
    static bool attr_done[2][64] = {};
    const bool paired = (a.group % 2 == 0);
    const int smem = (paired ? PairSmem::bytes : Smem::bytes) + 1024;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[paired][dev]) {
        cudaError_t e = paired ? cudaFuncSetAttribute(prefill_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                      smem)
                               : cudaFuncSetAttribute(prefill_causal_kernel,
                                                      cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        attr_done[paired][dev] = true;
    }
    const long long nqt = (a.S + kBM - 1) / kBM;
    const long long grid = nqt * a.B * (paired ? a.Hq / 2 : a.Hq);
    if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
    if (paired)
        prefill_pair_kernel<<<(unsigned)grid, kPairThreads, smem, stream>>>(tmQ, tmK, tmV, a);
    else
        prefill_causal_kernel<<<(unsigned)grid, kThreads, smem, stream>>>(tmQ, tmK, tmV, a);
    return cudaGetLastError();
}

}  // namespace gqa
