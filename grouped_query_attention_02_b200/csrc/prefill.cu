// prefill.cu -- causal GQA prefill on the tcgen05 tensor cores.
//
// One CTA computes two 128-row query tiles that read the same KV head: the
// query head h reads KV head h / g ("grouped-query and multi-query attention",
// study.greatitself.com: consecutive groups), K/V tiles are fetched by TMA once
// for both, and the CTAs of one group are neighbours so that a tile read from
// HBM serves the whole group out of L2.  The causal mask of anrans.github.io
// attention-variants ("Kernels do not need to copy the KV heads": lower
// triangle, diagonal included) is applied inside the diagonal tile only; tiles
// above the diagonal are never visited.
//
// The running maximum is only moved when a row's new maximum exceeds it by
// more than 8 (in log2 units); otherwise the weights are taken against the old
// maximum (they stay below 2^8, exact in fp32) and the O accumulator in TMEM
// needs no rescale.  The final division by l uses the same maximum, so the
// result is the same softmax.
#include "internal.h"
#include "ptx.cuh"

namespace gqa {

namespace {

constexpr int kD = kHeadDim;
constexpr int kBM = 128;                   // query rows per CTA
constexpr int kBN = 128;                   // keys per KV tile
constexpr int kTileBytes = kBM * kD * 2;   // 32 KB: one 128 x 128 bf16 tile
constexpr int kHalfTile = kTileBytes / 2;  // one 64-column half
constexpr int kSoftmaxThreads = 128;
constexpr uint32_t kTmemCols = 512;        // S0, S1, O (128 columns each), rounded to a power of two
constexpr float kRescaleThreshold = 8.0f;  // log2 units

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

// ----------------------------------------------------------------------------
// Paired variant: one CTA computes two 128-row query tiles ("streams") that
// read the same KV head, so every K/V tile in shared memory serves both.  For
// even group sizes the streams are the same query tile of two heads of one
// group (h, h+1), with the same causal shape; for odd group sizes (MHA
// included) they are query tiles 2k and 2k+1 of one head, which share key
// tiles 0..2k (the second stream has one more, its own diagonal).  Two softmax
// warpgroups (one per stream) alternate on the tensor core: while one works
// through its softmax, the MMAs of the other run.  Each warpgroup's P goes
// back into tensor memory over its own S (bf16, two per 32-bit column) and the
// PV product reads it from there, so both Q tiles and a two-stage K/V ring fit
// in shared memory.
//
// Warps: 0..3 softmax of stream 0, 4..7 softmax of stream 1 (TMEM lane quarter =
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

    // heaviest work first; the head pairs of one group (or the heads of one group) are neighbours
    const int nqt = (a.S + kBM - 1) / kBM;
    const int id = blockIdx.x;
    int b, hw[2], qtw[2];
    if (a.group % 2 == 0) {
        const int pairs = a.Hq / 2;
        const int per_qt = a.B * pairs;
        const int qt = nqt - 1 - id / per_qt;
        const int rem = id % per_qt;
        b = rem / pairs;
        hw[0] = 2 * (rem % pairs);
        hw[1] = hw[0] + 1;
        qtw[0] = qtw[1] = qt;
    } else {
        const int per_k = a.B * a.Hq;
        const int k = (nqt + 1) / 2 - 1 - id / per_k;
        const int rem = id % per_k;
        b = rem / a.Hq;
        hw[0] = hw[1] = rem % a.Hq;
        qtw[0] = 2 * k;
        qtw[1] = 2 * k + 1 < nqt ? 2 * k + 1 : -1;   // the last tile of an odd count has no partner
    }
    const int kvh = hw[0] / a.group;
    const int nt0 = qtw[0] + 1, nt1 = qtw[1] + 1;     // key tiles of each stream (0: stream absent)
    const int ntiles = nt0 > nt1 ? nt0 : nt1;
    auto ntw = [&](int w) { return w ? nt1 : nt0; };

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
            mbar_arrive_expect_tx(&bar[PQ_FULL], (nt1 > 0 ? 2 : 1) * kTileBytes);
            for (int w = 0; w < 2; ++w) {
                if (ntw(w) == 0) continue;
                uint8_t *qs = smem + PairSmem::q + w * kTileBytes;
                const int hq = w ? hw[1] : hw[0], q0 = (w ? qtw[1] : qtw[0]) * kBM;
                tma_load_4d(qs, &tmQ, &bar[PQ_FULL], 0, hq, q0, b);
                tma_load_4d(qs + kHalfTile, &tmQ, &bar[PQ_FULL], 64, hq, q0, b);
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
                for (int w = 0; w < 2; ++w)
                    if (ntw(w) > 0) issue_s(w, 0);
            }
            int pv_done = 0;
            for (int j = 0; ok && j < ntiles; ++j) {
                const int s = j & 1;
                const uint32_t v_addr = smem_u32(smem + PairSmem::kv + s * 2 * kTileBytes + kTileBytes);
                bool v_seen = false, k_next_seen = false;
                for (int w = 0; w < 2; ++w) {
                    if (j >= ntw(w)) continue;   // this stream's key tiles end before j
                    if (!wait_or_fail(&bar[PP_FULL + w], j & 1, a, err)) { ok = false; break; }
                    if (!v_seen && !wait_or_fail(&bar[PV_FULL + s], (j >> 1) & 1, a, err)) { ok = false; break; }
                    v_seen = true;
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < kBN / 16; ++ks) {
                        // A = P: 16 keys = 8 columns of packed bf16 pairs; B = V rows ks*16 .. +16
                        umma_ts(tmem + 256 + w * 128, tmem + w * 128 + ks * 8,
                                     desc_mnmajor(v_addr + ks * 2048, kHalfTile), idesc_o,
                                     (j > 0 || ks > 0) ? 1u : 0u);
                    }
                    if (j + 1 < ntw(w)) {
                        if (!k_next_seen && !wait_or_fail(&bar[PK_FULL + ((j + 1) & 1)], ((j + 1) >> 1) & 1, a, err)) {
                            ok = false;
                            break;
                        }
                        k_next_seen = true;
                        tc_fence_after();
                        issue_s(w, j + 1);
                    }
                }
                if (!ok) break;
                // the tile's last reader has been issued
                umma_commit(&bar[PKV_EMPTY + s]);
                ++pv_done;
            }
            if (ok && pv_done == ntiles) umma_commit(&bar[PO_FULL]);
            umma_commit(&bar[PDRAIN]);
            mbar_wait(&bar[PDRAIN], 0, a.wait_budget_ns);
        }
    } else {
        // ---------------- softmax warpgroup w: stream w (head hw[w], query tile qtw[w]), thread owns query row r
        const int w = warp >> 2;
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t tS = tmem + w * 128 + lane_off;
        const uint32_t tO = tmem + 256 + w * 128 + lane_off;
        const int qtile = w ? qtw[1] : qtw[0];
        const int qrow = qtile * kBM + r;
        const int hq = w ? hw[1] : hw[0];
        const int nt = ntw(w);
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = nt > 0;
        for (int j = 0; ok && j < nt; ++j) {
            if (!wait_or_fail(&bar[PS_FULL + w], j & 1, a, err)) { ok = false; break; }
            tc_fence_after();
            const bool diag = (j == qtile);
            // the row's 128 raw scores, loaded once (keys after the row hidden on the diagonal)
            uint32_t sr[128];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sr + c * 32);
            tmem_wait_ld();
            if (diag) {
#pragma unroll
                for (int i = 0; i < 128; ++i)
                    if (i > r) sr[i] = __float_as_uint(-INFINITY);
            }
            // the row maximum: three-input max, four independent partial maxima
            float pm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int i = 0; i < 128; i += 8) {
                pm[0] = fmax3(pm[0], __uint_as_float(sr[i + 0]), __uint_as_float(sr[i + 1]));
                pm[1] = fmax3(pm[1], __uint_as_float(sr[i + 2]), __uint_as_float(sr[i + 3]));
                pm[2] = fmax3(pm[2], __uint_as_float(sr[i + 4]), __uint_as_float(sr[i + 5]));
                pm[3] = fmax3(pm[3], __uint_as_float(sr[i + 6]), __uint_as_float(sr[i + 7]));
            }
            const float mraw = fmaxf(fmax3(pm[0], pm[1], pm[2]), pm[3]);
            const float m_new = fmaxf(m_run, mraw * a.qscale);
            const bool move = (m_new > m_run + kRescaleThreshold);
            const float m_use = move ? m_new : m_run;
            const float alpha = move ? ex2(m_run - m_new) : 1.f;
            // p = 2^(raw*qscale - m_use), summed, packed to bf16 pairs over S columns 0..63
            const float2 sc2 = make_float2(a.qscale, a.qscale);
            const float2 nm2 = make_float2(-m_use, -m_use);
            float2 ps[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                            make_float2(0.f, 0.f)};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    const float2 e = __ffma2_rn(
                        make_float2(__uint_as_float(sr[h * 32 + i]), __uint_as_float(sr[h * 32 + i + 1])), sc2, nm2);
                    const float2 pe = make_float2(ex2(e.x), ex2(e.y));
                    ps[(i >> 1) & 3] = __fadd2_rn(ps[(i >> 1) & 3], pe);
                    pk[i >> 1] = pack_bf16x2(pe.x, pe.y);
                }
                tmem_st16(tS + h * 16, pk);
            }
            // O holds tiles < j (the S_FULL commit covers the previous PV): rescale when the max moved;
            // PV of this tile is issued only after P_FULL below
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
                a.lse[((size_t)b * a.Hq + hq) * a.S + qrow] = (m_run + __log2f(l_run)) * 0.6931471805599453f;
            __nv_bfloat16 *orow_g = a.out + (((size_t)b * a.S + qrow) * a.Hq + hq) * kD;
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
    static bool attr_done[64] = {};
    const int smem = PairSmem::bytes + 1024;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(prefill_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        attr_done[dev] = true;
    }
    // even groups: (query tile, sequence, head pair); odd groups: (query-tile pair, sequence, head)
    const long long nqt = (a.S + kBM - 1) / kBM;
    const long long grid = a.group % 2 == 0 ? nqt * a.B * (a.Hq / 2) : ((nqt + 1) / 2) * a.B * a.Hq;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
    prefill_pair_kernel<<<(unsigned)grid, kPairThreads, smem, stream>>>(tmQ, tmK, tmV, a);
    return cudaGetLastError();
}

}  // namespace gqa
