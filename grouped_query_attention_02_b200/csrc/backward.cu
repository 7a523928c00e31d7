// backward.cu -- causal GQA prefill backward on the tcgen05 tensor cores.
//
// The gradients of a loss through O = softmax(scale Q K^T + causal mask) V, per query head h and its
// KV head h / g ("grouped-query and multi-query attention", study.greatitself.com, training
// paragraph: a shared key or value tensor receives the gradient of every query head of its group):
//
//   P = exp(scale q.k - lse)            (lse: the forward's log-sum-exp of the row)
//   dP = dO V^T,  D = rowsum(dO * O),   dS = P * (dP - D)
//   dV = sum over the group of P^T dO,  dK = scale * sum over the group of dS^T Q,  dQ = scale * dS K
//
// Two kernels, the dQ kernel first:
//   bwd_dkdv_kernel     one CTA per (sequence, KV head, 128-key tile): loops over the g query heads
//                       of the group and over the query tiles at or after the key tile; S^T = K Q^T and
//                       dP^T = V dO^T into tensor memory, P^T and dS^T back into tensor memory as bf16,
//                       then dV += P^T dO and dK += dS^T Q with the accumulators resident in tensor
//                       memory for the whole loop, so the group sum costs nothing extra
//   bwd_dq_kernel       one CTA per (sequence, query head, 128-row tile): first D = rowsum(dO * O) of
//                       its rows (left in the workspace for the dK/dV kernel), then a loop over the key
//                       tiles up to the diagonal: S = Q K^T and dP = dO V^T, dS back into tensor memory,
//                       then dQ += dS K
//
// Roles in both kernels (320 threads): warps 0..7 elementwise in two warpgroups of 64 columns each (one
// TMEM lane per thread: a key row of S^T in the dK/dV kernel, a query row of S in the dQ kernel),
// warp 8 TMA producer, warp 9 TMEM allocator + MMA issuer.  The probabilities and dS are rounded to bf16 for the products, as the
// forward rounds P.  Every wait is bounded; a kernel that gives up records GQA_ERR_DEVICE_TIMEOUT.
#include "internal.h"
#include "ptx.cuh"

namespace gqa {

namespace {

constexpr int kD = kHeadDim;
constexpr int kB = 128;                    // rows of a query tile and of a key tile
constexpr int kTile = kB * kD * 2;         // 32 KB: one 128 x 128 bf16 tile
constexpr int kHalf = kTile / 2;           // one 64-column half (128-byte rows, 128-byte swizzle)
constexpr int kThreads = 320;
constexpr int kEw = 256;                   // elementwise threads: two warpgroups, 64 columns each
constexpr int kProducerWarp = 8, kMmaWarp = 9;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ void record_status(int *status, int code)
{
    if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ bool wait_or_fail(uint64_t *bar, uint32_t parity, const BackwardArgs &a,
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

__device__ __forceinline__ uint64_t desc_kmajor(uint32_t saddr) { return umma_smem_desc(saddr, 16, 1024, 2); }
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t saddr) { return umma_smem_desc(saddr, kHalf, 1024, 2); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// ------------------------------------------------------------------------------------------------
// dK, dV
struct KvSmem {
    static constexpr int k = 0;                      // K tile of this CTA's keys
    static constexpr int v = k + kTile;              // V tile
    static constexpr int q = v + kTile;              // Q[2] tiles of the current / next query tile
    static constexpr int dout = q + 2 * kTile;       // dO[2]
    static constexpr int lse = dout + 2 * kTile;     // [2][128] floats: lse * log2(e) (+inf past the end)
    // (written by the first elementwise warpgroup; D below by the second)
    static constexpr int dsum = lse + 2 * kB * 4;    // [2][128] floats: D
    static constexpr int bars = dsum + 2 * kB * 4;
    static constexpr int nbars = 20;
    static constexpr int tmem_slot = bars + nbars * 8;
    static constexpr int err = tmem_slot + 8;
    static constexpr int bytes = err + 8;
};
// S^T and dP^T products complete (ST_FULL, DPT_FULL); P^T written (P_READY); dS^T written (DST_READY);
// (slots 13 and 14 are unused: the products that overwrite P^T and dS^T follow their readers in issue order)
// ST_READ / DPT_READ: the first elementwise warpgroup has read the raw columns the second one's packed
// output lands on
// RS_FULL: the row statistics of an iteration are in shared memory (the elementwise threads load them one
// iteration ahead, so their global-memory latency hides behind a whole iteration)
enum KvBar { KV_FULL = 0, QD_FULL = 1, QD_EMPTY = 3, RS_FULL = 5, ST_FULL = 9, DPT_FULL = 10,
             P_READY = 11, DST_READY = 12, ACC_FULL = 15, KDRAIN = 16, ST_READ = 17,
             DPT_READ = 18 };

__global__ void __launch_bounds__(kThreads, 1)
bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                const BackwardArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + KvSmem::bars);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + KvSmem::tmem_slot);
    volatile int *err = reinterpret_cast<volatile int *>(smem + KvSmem::err);

    // the key tiles near the start of a sequence have the most query tiles after them: first
    const int nt = (a.S + kB - 1) / kB;
    const int bk_count = a.B * a.Hkv;
    const int kt = blockIdx.x / bk_count;
    const int bk = blockIdx.x % bk_count;
    const int b = bk / a.Hkv, kvh = bk % a.Hkv;
    const int g = a.group;
    const int nq = nt - kt;                 // query tiles kt .. nt-1
    // (head, query tile) iterations: query tiles from the last down to kt, the group's heads innermost,
    // so that the CTAs of one KV head, which start together, read the same query and dO tiles at the
    // same time and L2 serves all but the first of them
    const int n_it = g * nq;
    const int k0 = kt * kB;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(&bar[KV_FULL], 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar[QD_FULL + s], 1);
            mbar_init(&bar[QD_EMPTY + s], 1);
            mbar_init(&bar[RS_FULL + s], kEw);
        }
        mbar_init(&bar[ST_FULL], 1);
        mbar_init(&bar[DPT_FULL], 1);
        mbar_init(&bar[P_READY], kEw);
        mbar_init(&bar[DST_READY], kEw);
        mbar_init(&bar[ACC_FULL], 1);
        mbar_init(&bar[KDRAIN], 1);
        mbar_init(&bar[ST_READ], kEw / 2);
        mbar_init(&bar[DPT_READ], kEw / 2);
        *err = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem, tdP = tmem + 128, tdV = tmem + 256, tdK = tmem + 384;

    if (warp == kProducerWarp) {
        // ---------------- producer: K, V once; then the Q, dO tiles of every iteration (TMA)
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            tma_prefetch_desc(&tmDO);
            mbar_arrive_expect_tx(&bar[KV_FULL], 2 * kTile);
            tma_load_4d(smem + KvSmem::k, &tmK, &bar[KV_FULL], 0, kvh, k0, b);
            tma_load_4d(smem + KvSmem::k + kHalf, &tmK, &bar[KV_FULL], 64, kvh, k0, b);
            tma_load_4d(smem + KvSmem::v, &tmV, &bar[KV_FULL], 0, kvh, k0, b);
            tma_load_4d(smem + KvSmem::v + kHalf, &tmV, &bar[KV_FULL], 64, kvh, k0, b);
            int issued = 0;
            for (int n = 0; n < n_it; ++n) {
                const int h = kvh * g + n % g, q0 = (nt - 1 - n / g) * kB, s = n & 1;
                if (n >= 2 && !wait_or_fail(&bar[QD_EMPTY + s], ((n >> 1) - 1) & 1, a, err)) break;
                mbar_arrive_expect_tx(&bar[QD_FULL + s], 2 * kTile);
                uint8_t *qs = smem + KvSmem::q + s * kTile, *ds = smem + KvSmem::dout + s * kTile;
                tma_load_4d(qs, &tmQ, &bar[QD_FULL + s], 0, h, q0, b);
                tma_load_4d(qs + kHalf, &tmQ, &bar[QD_FULL + s], 64, h, q0, b);
                tma_load_4d(ds, &tmDO, &bar[QD_FULL + s], 0, h, q0, b);
                tma_load_4d(ds + kHalf, &tmDO, &bar[QD_FULL + s], 64, h, q0, b);
                issued = n + 1;
            }
            // leave no copy in flight
            mbar_wait(&bar[KV_FULL], 0, a.wait_budget_ns);
            for (int n = issued - 1; n >= 0 && n >= issued - 2; --n)
                mbar_wait(&bar[QD_FULL + (n & 1)], (n >> 1) & 1, a.wait_budget_ns);
        }
    } else if (warp == kMmaWarp) {
        // ---------------- MMA issuer.  The elementwise pass hands over P^T before it computes dS^T, so
        // dV += P^T dO runs while dS^T is being formed, and the next S^T is issued right behind that dV
        // product (it overwrites the P^T columns dV reads; tcgen05 products of a CTA run in issue order),
        // so that the next iteration's scores are ready when the elementwise threads finish dS^T.  Per
        // iteration: dP^T(n), dV(n), S^T(n+1), dK(n).
        if (lane == 0) {
            const uint32_t idesc_s = umma_idesc_bf16(kB, kB, 0, 0);   // K (K-major) x Q (K-major) -> S^T
            const uint32_t idesc_g = umma_idesc_bf16(kB, kD, 0, 1);   // P^T / dS^T (TMEM) x dO / Q (MN-major)
            const uint32_t k_addr = smem_u32(smem + KvSmem::k), v_addr = smem_u32(smem + KvSmem::v);
            auto issue_st = [&](int n) {
                const uint32_t q_addr = smem_u32(smem + KvSmem::q + (n & 1) * kTile);
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * kHalf + (ks & 3) * 32;
                    umma_ss(tS, desc_kmajor(k_addr + off), desc_kmajor(q_addr + off), idesc_s, ks > 0 ? 1u : 0u);
                }
                umma_commit(&bar[ST_FULL]);
            };
            bool ok = wait_or_fail(&bar[KV_FULL], 0, a, err) && wait_or_fail(&bar[QD_FULL], 0, a, err);
            if (ok) {
                tc_fence_after();
                issue_st(0);
            }
            int done = 0;
            for (int n = 0; ok && n < n_it; ++n) {
                const int s = n & 1;
                const uint32_t q_addr = smem_u32(smem + KvSmem::q + s * kTile);
                const uint32_t o_addr = smem_u32(smem + KvSmem::dout + s * kTile);
                // dP^T: its columns held the previous dS^T, read by the previous dK product (issued before)
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * kHalf + (ks & 3) * 32;
                    umma_ss(tdP, desc_kmajor(v_addr + off), desc_kmajor(o_addr + off), idesc_s, ks > 0 ? 1u : 0u);
                }
                umma_commit(&bar[DPT_FULL]);
                // dV += P^T dO: A from tensor memory (16 query columns = 8 packed columns)
                if (!wait_or_fail(&bar[P_READY], n & 1, a, err)) break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < kB / 16; ++ks)
                    umma_ts(tdV, tS + ks * 8, desc_mnmajor(o_addr + ks * 2048), idesc_g, (n > 0 || ks > 0) ? 1u : 0u);
                // the next iteration's S^T, behind this dV product
                if (n + 1 < n_it) {
                    if (!wait_or_fail(&bar[QD_FULL + (s ^ 1)], ((n + 1) >> 1) & 1, a, err)) break;
                    tc_fence_after();
                    issue_st(n + 1);
                }
                // dK += dS^T Q
                if (!wait_or_fail(&bar[DST_READY], n & 1, a, err)) break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < kB / 16; ++ks)
                    umma_ts(tdK, tdP + ks * 8, desc_mnmajor(q_addr + ks * 2048), idesc_g, (n > 0 || ks > 0) ? 1u : 0u);
                umma_commit(&bar[QD_EMPTY + s]);
                done = n + 1;
            }
            if (done == n_it) umma_commit(&bar[ACC_FULL]);
            umma_commit(&bar[KDRAIN]);
            mbar_wait(&bar[KDRAIN], 0, a.wait_budget_ns);
        }
    } else {
        // ---------------- elementwise: thread t owns key k0 + t (TMEM lane t of S^T, dP^T, dV, dK);
        // warpgroup w takes query columns 64w .. 64w + 63
        const int w = warp >> 2;
        const int quarter = warp & 3;
        const int t = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        bool ok = true;
        const float2 qs2 = make_float2(a.qscale, a.qscale);
        // row statistic t of iteration n's query tile: lse * log2(e) (warpgroup 0) or D (warpgroup 1); rows
        // past the sequence get lse = +inf (P = 0) and D = 0
        auto row_stat = [&](int n) -> float {
            const int h = kvh * g + n % g, r = (nt - 1 - n / g) * kB + t;
            const size_t i = ((size_t)b * a.Hq + h) * a.S + r;
            return w == 0 ? (r < a.S ? a.lse[i] * kLog2e : INFINITY) : (r < a.S ? a.dsum[i] : 0.f);
        };
        float *stat_smem = reinterpret_cast<float *>(smem + (w == 0 ? KvSmem::lse : KvSmem::dsum));
        stat_smem[t] = row_stat(0);
        mbar_arrive(&bar[RS_FULL]);
        for (int n = 0; n < n_it; ++n) {
            const int s = n & 1;
            const bool diag = n / g == nq - 1;    // the query tile that holds this CTA's keys (the last)
            if (!wait_or_fail(&bar[RS_FULL + s], (n >> 1) & 1, a, err)) { ok = false; break; }
            // the next iteration's statistic, in flight during this iteration
            const float next_stat = n + 1 < n_it ? row_stat(n + 1) : 0.f;
            if (!wait_or_fail(&bar[ST_FULL], n & 1, a, err)) { ok = false; break; }
            tc_fence_after();
            const float *ls = reinterpret_cast<const float *>(smem + KvSmem::lse) + s * kB + w * 64;
            const float *dd = reinterpret_cast<const float *>(smem + KvSmem::dsum) + s * kB + w * 64;
            // pass 1: P^T = 2^(s qscale - lse2) over this warpgroup's 64 columns, kept in registers and
            // written back as bf16 (packed: columns 64w.. land on packed columns 32w..)
            float p[64];
            {
                uint32_t sr[64];
                tmem_ld32(tS + lane_off + w * 64, sr);
                tmem_ld32(tS + lane_off + w * 64 + 32, sr + 32);
                tmem_wait_ld();
                if (w == 0) mbar_arrive(&bar[ST_READ]);
                if (diag) {
                    // query c of the tile sees key t only when c >= t on the diagonal tile (weight 2^-inf = 0);
                    // masked before the loop below, which then has no branch
#pragma unroll
                    for (int i = 0; i < 64; ++i)
                        if (w * 64 + i < t) sr[i] = __float_as_uint(-INFINITY);
                }
                const float4 *ls4 = reinterpret_cast<const float4 *>(ls);
                uint32_t pw[32];
#pragma unroll
                for (int i = 0; i < 64; i += 4) {
                    const float4 l = ls4[i >> 2];
                    const float2 x01 = __ffma2_rn(make_float2(__uint_as_float(sr[i]), __uint_as_float(sr[i + 1])),
                                                  qs2, make_float2(-l.x, -l.y));
                    const float2 x23 = __ffma2_rn(make_float2(__uint_as_float(sr[i + 2]), __uint_as_float(sr[i + 3])),
                                                  qs2, make_float2(-l.z, -l.w));
                    p[i] = ex2(x01.x);
                    p[i + 1] = ex2(x01.y);
                    p[i + 2] = ex2(x23.x);
                    p[i + 3] = ex2(x23.y);
                    pw[i >> 1] = pack_bf16x2(p[i], p[i + 1]);
                    pw[(i >> 1) + 1] = pack_bf16x2(p[i + 2], p[i + 3]);
                }
                // the second warpgroup's packed columns 32..63 are raw columns the first one reads
                if (w == 1 && !wait_or_fail(&bar[ST_READ], n & 1, a, err)) { ok = false; break; }
                tmem_st32(tS + lane_off + w * 32, pw);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bar[P_READY]);
            // pass 2: dS^T = P^T (dP^T - D), written back as bf16 over dP^T
            if (!wait_or_fail(&bar[DPT_FULL], n & 1, a, err)) { ok = false; break; }
            tc_fence_after();
            {
                uint32_t pr[64];
                tmem_ld32(tdP + lane_off + w * 64, pr);
                tmem_ld32(tdP + lane_off + w * 64 + 32, pr + 32);
                tmem_wait_ld();
                if (w == 0) mbar_arrive(&bar[DPT_READ]);
                const float4 *dd4 = reinterpret_cast<const float4 *>(dd);
                uint32_t dw[32];
#pragma unroll
                for (int i = 0; i < 64; i += 4) {
                    const float4 dv = dd4[i >> 2];
                    const float2 s01 = __fmul2_rn(make_float2(p[i], p[i + 1]),
                                                  __fadd2_rn(make_float2(__uint_as_float(pr[i]), __uint_as_float(pr[i + 1])),
                                                             make_float2(-dv.x, -dv.y)));
                    const float2 s23 = __fmul2_rn(make_float2(p[i + 2], p[i + 3]),
                                                  __fadd2_rn(make_float2(__uint_as_float(pr[i + 2]), __uint_as_float(pr[i + 3])),
                                                             make_float2(-dv.z, -dv.w)));
                    dw[i >> 1] = pack_bf16x2(s01.x, s01.y);
                    dw[(i >> 1) + 1] = pack_bf16x2(s23.x, s23.y);
                }
                if (w == 1 && !wait_or_fail(&bar[DPT_READ], n & 1, a, err)) { ok = false; break; }
                tmem_st32(tdP + lane_off + w * 32, dw);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bar[DST_READY]);
            // the other buffer was read in iteration n - 1, which both warpgroups have left: the dP^T of
            // this iteration needed the dK product of n - 1, which needed every thread's dS^T of n - 1
            if (n + 1 < n_it) {
                stat_smem[(s ^ 1) * kB + t] = next_stat;
                mbar_arrive(&bar[RS_FULL + (s ^ 1)]);
            }
        }
        if (ok && wait_or_fail(&bar[ACC_FULL], 0, a, err)) {
            tc_fence_after();
            const int key = k0 + t;
            __nv_bfloat16 *dvg = a.dv + (((size_t)b * a.S + key) * a.Hkv + kvh) * kD;
            __nv_bfloat16 *dkg = a.dk + (((size_t)b * a.S + key) * a.Hkv + kvh) * kD;
#pragma unroll 1
            for (int c = 2 * w; c < 2 * w + 2; ++c) {
                uint32_t vr[32], kr[32];
                tmem_ld32(tdV + lane_off + c * 32, vr);
                tmem_ld32(tdK + lane_off + c * 32, kr);
                tmem_wait_ld();
                if (key < a.S) {
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        uint4 v4;
                        v4.x = pack_bf16x2(__uint_as_float(vr[i + 0]), __uint_as_float(vr[i + 1]));
                        v4.y = pack_bf16x2(__uint_as_float(vr[i + 2]), __uint_as_float(vr[i + 3]));
                        v4.z = pack_bf16x2(__uint_as_float(vr[i + 4]), __uint_as_float(vr[i + 5]));
                        v4.w = pack_bf16x2(__uint_as_float(vr[i + 6]), __uint_as_float(vr[i + 7]));
                        *reinterpret_cast<uint4 *>(dvg + c * 32 + i) = v4;
                        v4.x = pack_bf16x2(__uint_as_float(kr[i + 0]) * a.scale, __uint_as_float(kr[i + 1]) * a.scale);
                        v4.y = pack_bf16x2(__uint_as_float(kr[i + 2]) * a.scale, __uint_as_float(kr[i + 3]) * a.scale);
                        v4.z = pack_bf16x2(__uint_as_float(kr[i + 4]) * a.scale, __uint_as_float(kr[i + 5]) * a.scale);
                        v4.w = pack_bf16x2(__uint_as_float(kr[i + 6]) * a.scale, __uint_as_float(kr[i + 7]) * a.scale);
                        *reinterpret_cast<uint4 *>(dkg + c * 32 + i) = v4;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------------------------------------
// dQ
struct QSmem {
    static constexpr int q = 0;                      // this CTA's Q tile
    static constexpr int dout = q + kTile;           // and its dO tile
    // separate rings: K is read by S and by the dQ product, V only by dP, which frees it much earlier
    static constexpr int kstages = 3, vstages = 2;
    static constexpr int k = dout + kTile;           // K[3] tiles
    static constexpr int v = k + kstages * kTile;    // V[2] tiles
    static constexpr int bars = v + vstages * kTile;
    static constexpr int nbars = 24;
    static constexpr int tmem_slot = bars + nbars * 8;
    static constexpr int err = tmem_slot + 8;
    static constexpr int bytes = err + 8;
};
// S2_FULL / S2_FREE / DS_READY: per S buffer (the pass of tile j + 1 can finish before the issuer has
// seen tile j's, so DS_READY alternates like the buffers); DP_FREE: the pass has dP in registers
enum QBar { QO_FULL = 0, K2_FULL = 1, K2_EMPTY = 4, S2_FULL = 7, S2_FREE = 9, DP_FULL = 11, DP_FREE = 12,
            DS_READY = 13, DQ_FULL = 15, QDRAIN = 16, V2_FULL = 18, V2_EMPTY = 20,
            // per S buffer: the first warpgroup has read the raw columns the second one packs its dS onto (see
            // the dK/dV kernel's ST_READ).  One barrier per buffer: S is double-buffered, so the first
            // warpgroup can read the next tile's S before the second looks at this tile's phase; reading S of
            // tile j + 2 needs the dS of tile j from both warpgroups, so per buffer no phase is passed unseen
            S2_READ = 22 };
static_assert(V2_EMPTY + QSmem::vstages <= S2_READ && S2_READ + 2 <= QSmem::nbars && K2_FULL + QSmem::kstages <= K2_EMPTY &&
                  K2_EMPTY + QSmem::kstages <= S2_FULL && DPT_READ < KvSmem::nbars, "barrier slots");

__global__ void __launch_bounds__(kThreads, 1)
bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
              const BackwardArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + QSmem::bars);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + QSmem::tmem_slot);
    volatile int *err = reinterpret_cast<volatile int *>(smem + QSmem::err);

    // the last query tiles see the most key tiles: first
    const int nt = (a.S + kB - 1) / kB;
    const int bh_count = a.B * a.Hq;
    const int qt = nt - 1 - blockIdx.x / bh_count;
    const int bh = blockIdx.x % bh_count;
    const int b = bh / a.Hq, h = bh % a.Hq;
    const int kvh = h / a.group;
    const int q0 = qt * kB;
    const int ntiles = qt + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(&bar[QO_FULL], 1);
        for (int s = 0; s < QSmem::kstages; ++s) {
            mbar_init(&bar[K2_FULL + s], 1);
            mbar_init(&bar[K2_EMPTY + s], 1);
        }
        for (int s = 0; s < QSmem::vstages; ++s) {
            mbar_init(&bar[V2_FULL + s], 1);
            mbar_init(&bar[V2_EMPTY + s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar[S2_FULL + s], 1);
            mbar_init(&bar[S2_FREE + s], 1);
        }
        mbar_init(&bar[DP_FULL], 1);
        mbar_init(&bar[DP_FREE], kEw);
        mbar_init(&bar[DS_READY], kEw);
        mbar_init(&bar[DS_READY + 1], kEw);
        mbar_init(&bar[DQ_FULL], 1);
        mbar_init(&bar[QDRAIN], 1);
        for (int s = 0; s < 2; ++s) mbar_init(&bar[S2_READ + s], kEw / 2);
        *err = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // S[2] (dS is packed into the S buffer it came from), dP, the dQ accumulator
    const uint32_t tS0 = tmem, tdP = tmem + 256, tdQ = tmem + 384;

    if (warp == kProducerWarp) {
        // ---------------- producer: Q, dO once; K_j into a three-stage ring, V_j into a two-stage ring
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            tma_prefetch_desc(&tmDO);
            mbar_arrive_expect_tx(&bar[QO_FULL], 2 * kTile);
            tma_load_4d(smem + QSmem::q, &tmQ, &bar[QO_FULL], 0, h, q0, b);
            tma_load_4d(smem + QSmem::q + kHalf, &tmQ, &bar[QO_FULL], 64, h, q0, b);
            tma_load_4d(smem + QSmem::dout, &tmDO, &bar[QO_FULL], 0, h, q0, b);
            tma_load_4d(smem + QSmem::dout + kHalf, &tmDO, &bar[QO_FULL], 64, h, q0, b);
            int issued_k = 0, issued_v = 0;
            for (int j = 0; j < ntiles; ++j) {
                const int sk = j % QSmem::kstages, sv = j % QSmem::vstages;
                if (j >= QSmem::kstages &&
                    !wait_or_fail(&bar[K2_EMPTY + sk], ((j / QSmem::kstages) - 1) & 1, a, err))
                    break;
                uint8_t *ks = smem + QSmem::k + sk * kTile;
                mbar_arrive_expect_tx(&bar[K2_FULL + sk], kTile);
                tma_load_4d(ks, &tmK, &bar[K2_FULL + sk], 0, kvh, j * kB, b);
                tma_load_4d(ks + kHalf, &tmK, &bar[K2_FULL + sk], 64, kvh, j * kB, b);
                issued_k = j + 1;
                if (j >= QSmem::vstages &&
                    !wait_or_fail(&bar[V2_EMPTY + sv], ((j / QSmem::vstages) - 1) & 1, a, err))
                    break;
                uint8_t *vs = smem + QSmem::v + sv * kTile;
                mbar_arrive_expect_tx(&bar[V2_FULL + sv], kTile);
                tma_load_4d(vs, &tmV, &bar[V2_FULL + sv], 0, kvh, j * kB, b);
                tma_load_4d(vs + kHalf, &tmV, &bar[V2_FULL + sv], 64, kvh, j * kB, b);
                issued_v = j + 1;
            }
            // leave no copy in flight
            for (int j = issued_k - 1; j >= 0 && j >= issued_k - QSmem::kstages; --j)
                mbar_wait(&bar[K2_FULL + j % QSmem::kstages], (j / QSmem::kstages) & 1, a.wait_budget_ns);
            for (int j = issued_v - 1; j >= 0 && j >= issued_v - QSmem::vstages; --j)
                mbar_wait(&bar[V2_FULL + j % QSmem::vstages], (j / QSmem::vstages) & 1, a.wait_budget_ns);
            mbar_wait(&bar[QO_FULL], 0, a.wait_budget_ns);
        }
    } else if (warp == kMmaWarp) {
        // ---------------- MMA issuer.  S is double-buffered and dP is released as soon as the elementwise
        // pass holds it in registers, so the next tile's S and dP products run during this tile's pass.
        if (lane == 0) {
            const uint32_t idesc_s = umma_idesc_bf16(kB, kB, 0, 0);   // Q / dO (K-major) x K / V (K-major)
            const uint32_t idesc_q = umma_idesc_bf16(kB, kD, 0, 1);   // dS (TMEM) x K (MN-major)
            const uint32_t q_addr = smem_u32(smem + QSmem::q), o_addr = smem_u32(smem + QSmem::dout);
            bool ok = wait_or_fail(&bar[QO_FULL], 0, a, err);
            int done = 0;
            for (int j = 0; ok && j <= ntiles; ++j) {
                if (j < ntiles) {
                    const int s = j & 1, sk = j % QSmem::kstages, sv = j % QSmem::vstages;
                    if (!wait_or_fail(&bar[K2_FULL + sk], (j / QSmem::kstages) & 1, a, err)) break;
                    // this S buffer's previous dS is read by the dQ product of tile j - 2, issued before
                    tc_fence_after();
                    const uint32_t k_addr = smem_u32(smem + QSmem::k + sk * kTile);
                    const uint32_t v_addr = smem_u32(smem + QSmem::v + sv * kTile);
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks) {
                        const uint32_t off = (ks >> 2) * kHalf + (ks & 3) * 32;
                        umma_ss(tS0 + s * 128, desc_kmajor(q_addr + off), desc_kmajor(k_addr + off), idesc_s,
                                ks > 0 ? 1u : 0u);
                    }
                    umma_commit(&bar[S2_FULL + s]);
                    // the previous tile's dP is in the elementwise threads' registers by now
                    if (j >= 1 && !wait_or_fail(&bar[DP_FREE], (j - 1) & 1, a, err)) break;
                    if (!wait_or_fail(&bar[V2_FULL + sv], (j / QSmem::vstages) & 1, a, err)) break;
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks) {
                        const uint32_t off = (ks >> 2) * kHalf + (ks & 3) * 32;
                        umma_ss(tdP, desc_kmajor(o_addr + off), desc_kmajor(v_addr + off), idesc_s, ks > 0 ? 1u : 0u);
                    }
                    umma_commit(&bar[DP_FULL]);
                    umma_commit(&bar[V2_EMPTY + sv]);
                }
                if (j >= 1) {
                    const int jp = j - 1, s = jp & 1, sk = jp % QSmem::kstages;
                    if (!wait_or_fail(&bar[DS_READY + s], (jp >> 1) & 1, a, err)) break;
                    tc_fence_after();
                    const uint32_t k_addr = smem_u32(smem + QSmem::k + sk * kTile);
                    // dQ += dS K: A = dS from tensor memory (16 keys = 8 packed columns), B = K rows (MN-major)
#pragma unroll
                    for (int ks = 0; ks < kB / 16; ++ks)
                        umma_ts(tdQ, tS0 + s * 128 + ks * 8, desc_mnmajor(k_addr + ks * 2048), idesc_q,
                                (jp > 0 || ks > 0) ? 1u : 0u);
                    umma_commit(&bar[S2_FREE + s]);
                    umma_commit(&bar[K2_EMPTY + sk]);
                    done = j;
                }
            }
            if (done == ntiles) umma_commit(&bar[DQ_FULL]);
            umma_commit(&bar[QDRAIN]);
            mbar_wait(&bar[QDRAIN], 0, a.wait_budget_ns);
        }
    } else {
        // ---------------- elementwise: thread r owns query row q0 + r (TMEM lane r of S, dP, dQ);
        // warpgroup w takes key columns 64w .. 64w + 63
        const int w = warp >> 2;
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int qrow = q0 + r;
        const size_t rs = ((size_t)b * a.Hq + h) * a.S + qrow;
        const float lse2 = qrow < a.S ? a.lse[rs] * kLog2e : INFINITY;
        // D = rowsum(dO * O) of this row in fp32, from the dO tile in shared memory and the row of O in
        // global memory; the first warpgroup leaves it in the workspace for the dK/dV kernel, which runs next
        bool ok = wait_or_fail(&bar[QO_FULL], 0, a, err);
        float dsum = 0.f;
        if (ok && qrow < a.S) {
            const uint4 *orow = reinterpret_cast<const uint4 *>(a.out + (((size_t)b * a.S + qrow) * a.Hq + h) * kD);
            const uint8_t *grow = smem + QSmem::dout + r * 128;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    // the 128-byte swizzle: chunk c of row r sits at chunk c ^ (r % 8)
                    const uint4 gv = *reinterpret_cast<const uint4 *>(grow + hf * kHalf + ((c ^ (r & 7)) << 4));
                    const uint4 ov = orow[hf * 8 + c];
                    dsum += bf16_lo(gv.x) * bf16_lo(ov.x) + bf16_hi(gv.x) * bf16_hi(ov.x) + bf16_lo(gv.y) * bf16_lo(ov.y) +
                            bf16_hi(gv.y) * bf16_hi(ov.y) + bf16_lo(gv.z) * bf16_lo(ov.z) + bf16_hi(gv.z) * bf16_hi(ov.z) +
                            bf16_lo(gv.w) * bf16_lo(ov.w) + bf16_hi(gv.w) * bf16_hi(ov.w);
                }
            }
            if (w == 0) a.dsum[rs] = dsum;
        }
        const float2 qs2 = make_float2(a.qscale, a.qscale), nl2 = make_float2(-lse2, -lse2);
        const float2 nd2 = make_float2(-dsum, -dsum);
        for (int j = 0; ok && j < ntiles; ++j) {
            const int s = j & 1;
            // dP into registers first, then release it for the next tile's product
            if (!wait_or_fail(&bar[DP_FULL], j & 1, a, err)) { ok = false; break; }
            tc_fence_after();
            uint32_t pr[64];
            tmem_ld32(tdP + lane_off + w * 64, pr);
            tmem_ld32(tdP + lane_off + w * 64 + 32, pr + 32);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&bar[DP_FREE]);
            if (!wait_or_fail(&bar[S2_FULL + s], (j >> 1) & 1, a, err)) { ok = false; break; }
            tc_fence_after();
            const bool diag = (j == qt);
            const int kend = a.S - j * kB;        // keys of this tile that exist
            const bool edge = diag || kend < kB;  // masks only on the diagonal tile and at the sequence's end
            uint32_t sr[64];
            tmem_ld32(tS0 + s * 128 + lane_off + w * 64, sr);
            tmem_ld32(tS0 + s * 128 + lane_off + w * 64 + 32, sr + 32);
            tmem_wait_ld();
            if (w == 0) mbar_arrive(&bar[S2_READ + s]);
            if (edge) {
                // key c of the tile: after the row on the diagonal tile, or past the sequence (its weight
                // is 2^-inf = 0); masked before the loop below, which then has no branch
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    const int c = w * 64 + i;
                    if ((diag && c > r) || c >= kend) sr[i] = __float_as_uint(-INFINITY);
                }
            }
            uint32_t dw[32];
#pragma unroll
            for (int i = 0; i < 64; i += 2) {
                const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[i]), __uint_as_float(sr[i + 1])), qs2, nl2);
                const float2 p = make_float2(ex2(x.x), ex2(x.y));
                const float2 d = __fmul2_rn(p, __fadd2_rn(make_float2(__uint_as_float(pr[i]), __uint_as_float(pr[i + 1])), nd2));
                dw[i >> 1] = pack_bf16x2(d.x, d.y);
            }
            // packed: key columns 64w.. land on packed columns 32w.., which for w = 1 are raw columns the
            // first warpgroup reads
            if (w == 1 && !wait_or_fail(&bar[S2_READ + s], (j >> 1) & 1, a, err)) { ok = false; break; }
            tmem_st32(tS0 + s * 128 + lane_off + w * 32, dw);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bar[DS_READY + s]);
        }
        if (ok && wait_or_fail(&bar[DQ_FULL], 0, a, err)) {
            tc_fence_after();
            __nv_bfloat16 *dqg = a.dq + (((size_t)b * a.S + qrow) * a.Hq + h) * kD;
#pragma unroll 1
            for (int c = 2 * w; c < 2 * w + 2; ++c) {
                uint32_t qr[32];
                tmem_ld32(tdQ + lane_off + c * 32, qr);
                tmem_wait_ld();
                if (qrow < a.S) {
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        uint4 v4;
                        v4.x = pack_bf16x2(__uint_as_float(qr[i + 0]) * a.scale, __uint_as_float(qr[i + 1]) * a.scale);
                        v4.y = pack_bf16x2(__uint_as_float(qr[i + 2]) * a.scale, __uint_as_float(qr[i + 3]) * a.scale);
                        v4.z = pack_bf16x2(__uint_as_float(qr[i + 4]) * a.scale, __uint_as_float(qr[i + 5]) * a.scale);
                        v4.w = pack_bf16x2(__uint_as_float(qr[i + 6]) * a.scale, __uint_as_float(qr[i + 7]) * a.scale);
                        *reinterpret_cast<uint4 *>(dqg + c * 32 + i) = v4;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

cudaError_t launch_prefill_backward(const CUtensorMap &tmQ, const CUtensorMap &tmK, const CUtensorMap &tmV,
                                    const CUtensorMap &tmDO, const BackwardArgs &a, cudaStream_t stream,
                                    int *launches)
{
    static bool attr_done[64] = {};
    const int smem_kv = KvSmem::bytes + 1024, smem_q = QSmem::bytes + 1024;
    static_assert(KvSmem::bytes + 1024 <= 227 * 1024 && QSmem::bytes + 1024 <= 227 * 1024, "shared memory budget");
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(bwd_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_kv);
        if (e != cudaSuccess) return e;
        if ((e = cudaFuncSetAttribute(bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_q)) !=
            cudaSuccess)
            return e;
        attr_done[dev] = true;
    }
    const long long nt = (a.S + kB - 1) / kB;
    const long long grid_kv = nt * a.B * a.Hkv, grid_q = nt * a.B * a.Hq;
    if (grid_q > 0x7fffffffLL) return cudaErrorInvalidValue;
    // the dQ kernel first: it also forms D = rowsum(dO * O), which the dK/dV kernel reads
    bwd_dq_kernel<<<(unsigned)grid_q, kThreads, smem_q, stream>>>(tmQ, tmK, tmV, tmDO, a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    ++*launches;
    bwd_dkdv_kernel<<<(unsigned)grid_kv, kThreads, smem_kv, stream>>>(tmQ, tmK, tmV, tmDO, a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    ++*launches;
    return cudaSuccess;
}

}  // namespace gqa
