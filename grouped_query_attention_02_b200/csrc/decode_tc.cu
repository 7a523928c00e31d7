// decode_tc.cu -- GQA decode with the dot products on the tcgen05 tensor cores.
//
// Same contract as decode_split_kernel (one CTA per (sequence b, KV head,
// split), split partials merged by decode_combine_kernel), but the group's g
// query heads are the N dimension of two small matrix products per 128-token
// tile, with the tokens as the 128-row M dimension:
//
//   S^T [128 tokens x N] = K_tile [128 x d] . Q_g^T        (A = K, K-major; B = Q, K-major)
//   O^T [d x N]         += V_tile^T [d x 128] . P^T [128 x N]  (A = V, MN-major; B = P^T, MN-major)
//
// N is g rounded up to 16 or 32 (extra query rows are zero).  The softmax
// weights enter the second product as two bf16 terms (hi + lo), so the
// result carries them to about 2^-17 relative, like an fp32 weight.  Each K/V tile is
// fetched from HBM once by TMA and serves every head of the group ("Kernels do
// not need to copy the KV heads", anrans.github.io attention-variants: the
// group's query heads become extra rows against one shared KV head).
//
// The softmax runs on 128 threads, one token per thread (TMEM lane = token
// for S^T, lane = d for O^T).  The running maximum of each head is CTA-wide
// and only moves when some score exceeds it by more than 8 (log2 units); in
// the common case a tile costs one warp vote and one group barrier, no
// reduction.  When it moves, the tile maximum is reduced across the CTA, the
// per-thread partial sums and the O^T accumulator in TMEM are rescaled.
//
// Warps: 0..3 softmax + epilogue, 4 TMA producer, 5 TMEM allocator + MMA issuer.
#include "internal.h"
#include "ptx.cuh"

namespace gqa {

namespace {

constexpr int kD = kHeadDim;
constexpr int kTok = 128;                 // tokens per tile (the M of S^T)
constexpr int kTile = kTok * kD * 2;      // 32 KB: one K or V tile
constexpr int kHalf = kTile / 2;          // one 64-column half
constexpr int kThreads = 192;
constexpr int kSoftmax = 128;
constexpr float kMoveThreshold = 8.0f;

template <int N>
struct TcCfg {
    static constexpr int stages = 3;
    static constexpr int stage_bytes = 2 * kTile;             // K then V
    static constexpr int q_off = stages * stage_bytes;        // Q: [2 halves][N rows][128 B], swizzled
    static constexpr int q_half = N * 128;
    static constexpr int p_off = q_off + 2 * q_half;          // P^T hi, then lo: [N/8][16 token groups][8][8] bf16
    static constexpr int p_bytes = N * kTok * 2;
    static constexpr int red_off = p_off + 2 * p_bytes;       // [2][4][N] floats: tile maxima per warp
    static constexpr int lsum_off = red_off + 2 * 4 * N * 4;  // [4][N] floats: l partials per warp
    static constexpr int vote_off = lsum_off + 4 * N * 4;     // [2][4] ints
    static constexpr int bar_off = vote_off + 32;
    // barriers: k_full[3], v_full[3], kv_empty[3], s_full[2], s_free[2], p_full, p_free, o_full, drain, grp
    static constexpr int nbars = 18;
    static constexpr int tmem_off = bar_off + nbars * 8;
    static constexpr int err_off = tmem_off + 8;
    static constexpr int bytes = err_off + 8;
    static constexpr uint32_t tmem_cols = (3 * N <= 32) ? 32 : (3 * N <= 64 ? 64 : 128);
    static_assert(bytes + 1024 <= 227 * 1024, "shared memory budget");
};

enum : int { K_FULL = 0, V_FULL = 3, KV_EMPTY = 6, S_FULL = 9, S_FREE = 11, P_FULL = 13, P_FREE = 14, O_FULL = 15,
             DRAIN = 16, GRP = 17 };

__device__ __forceinline__ void record_status(int *status, int code)
{
    if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ bool wait_or_fail(uint64_t *bar, uint32_t parity, const DecodeArgs &a, volatile int *err)
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

// Barrier among the 128 softmax threads on an mbarrier, so that it gives up (bounded) like every other wait
// instead of blocking forever when another role has failed.  `uses` counts this thread's earlier syncs.
__device__ __forceinline__ bool group_sync(uint64_t *grp, int &uses, const DecodeArgs &a, volatile int *err)
{
    mbar_arrive(grp);
    const bool r = wait_or_fail(grp, uses & 1, a, err);
    ++uses;
    return r;
}

template <int N>
__device__ __forceinline__ void tmem_ld_row(uint32_t taddr, uint32_t (&r)[N])
{
    if constexpr (N == 16) {
        tmem_ld16(taddr, r);
    } else {
        uint32_t (&lo)[16] = *reinterpret_cast<uint32_t (*)[16]>(&r[0]);
        uint32_t (&hi)[16] = *reinterpret_cast<uint32_t (*)[16]>(&r[16]);
        tmem_ld16(taddr, lo);
        tmem_ld16(taddr + 16, hi);
    }
}

template <int N>
__device__ __forceinline__ void tmem_st_row(uint32_t taddr, const uint32_t (&r)[N])
{
    if constexpr (N == 16) {
        tmem_st16(taddr, r);
    } else {
        const uint32_t (&lo)[16] = *reinterpret_cast<const uint32_t (*)[16]>(&r[0]);
        const uint32_t (&hi)[16] = *reinterpret_cast<const uint32_t (*)[16]>(&r[16]);
        tmem_st16(taddr, lo);
        tmem_st16(taddr + 16, hi);
    }
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

template <int N>
__global__ void __launch_bounds__(kThreads, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, const DecodeArgs a)
{
    using C = TcCfg<N>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int split = blockIdx.x;
    const int kvh = blockIdx.y;
    const int b = blockIdx.z;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    int T = a.seqlens[b];
    T = T < 0 ? 0 : (T > a.Tmax ? a.Tmax : T);
    const int t_begin = split * a.chunk;
    const int t_end = min(t_begin + a.chunk, T);
    const int h0 = kvh * a.group;
    const int g = a.group;

    if (t_end <= t_begin) {
        if (a.nsplit == 1) {
            const uint4 z = make_uint4(0, 0, 0, 0);
            for (int i = threadIdx.x; i < g * (kD / 8); i += kThreads)
                reinterpret_cast<uint4 *>(a.out + ((size_t)b * a.Hq + h0) * kD)[i] = z;
        }
        return;
    }
    const int ntiles = (t_end - t_begin + kTok - 1) / kTok;

    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + C::bar_off);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::tmem_off);
    volatile int *err = reinterpret_cast<volatile int *>(smem + C::err_off);
    float *red = reinterpret_cast<float *>(smem + C::red_off);
    float *lsum = reinterpret_cast<float *>(smem + C::lsum_off);
    volatile int *vote = reinterpret_cast<volatile int *>(smem + C::vote_off);
    uint8_t *qs = smem + C::q_off;
    uint8_t *ps = smem + C::p_off;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::stages; ++s) {
            mbar_init(&bar[K_FULL + s], 1);
            mbar_init(&bar[V_FULL + s], 1);
            mbar_init(&bar[KV_EMPTY + s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar[S_FULL + s], 1);
            mbar_init(&bar[S_FREE + s], kSoftmax);
        }
        mbar_init(&bar[P_FULL], kSoftmax);
        mbar_init(&bar[P_FREE], 1);
        mbar_init(&bar[O_FULL], 1);
        mbar_init(&bar[DRAIN], 1);
        mbar_init(&bar[GRP], kSoftmax);
        *err = 0;
        fence_barrier_init();
    }
    // the group's query rows, bf16, K-major with the 128-byte swizzle; rows g..N-1 are zero
    for (int i = threadIdx.x; i < N * (kD / 8); i += kThreads) {
        const int n = i / (kD / 8), c16 = i % (kD / 8);        // row, 16-byte chunk of the 256-byte row
        uint4 v = make_uint4(0, 0, 0, 0);
        if (n < g) v = reinterpret_cast<const uint4 *>(a.q + ((size_t)b * a.Hq + h0 + n) * kD)[c16];
        const int half = c16 >> 3, c = c16 & 7;
        *reinterpret_cast<uint4 *>(qs + half * C::q_half + n * 128 + ((c ^ (n & 7)) << 4)) = v;
    }
    fence_proxy_async_smem();
    if (warp == 5) {
        tmem_alloc(tmem_slot, C::tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS[2] = {tmem, tmem + N};
    const uint32_t tO = tmem + 2 * N;

    if (warp == 4) {
        // ---------------- TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            int issued = 0;
            for (int j = 0; j < ntiles; ++j) {
                const int s = j % C::stages;
                if (j >= C::stages && !wait_or_fail(&bar[KV_EMPTY + s], ((j / C::stages) - 1) & 1, a, err)) break;
                uint8_t *ks = smem + s * C::stage_bytes;
                const int t0 = t_begin + j * kTok;
                mbar_arrive_expect_tx(&bar[K_FULL + s], kTile);
                tma_load_4d(ks, &tmK, &bar[K_FULL + s], 0, kvh, t0, b);
                tma_load_4d(ks + kHalf, &tmK, &bar[K_FULL + s], 64, kvh, t0, b);
                mbar_arrive_expect_tx(&bar[V_FULL + s], kTile);
                tma_load_4d(ks + kTile, &tmV, &bar[V_FULL + s], 0, kvh, t0, b);
                tma_load_4d(ks + kTile + kHalf, &tmV, &bar[V_FULL + s], 64, kvh, t0, b);
                ++issued;
            }
            for (int j = issued - 1; j >= 0 && j >= issued - C::stages; --j) {
                const uint32_t ph = (j / C::stages) & 1;
                mbar_wait(&bar[K_FULL + j % C::stages], ph, a.wait_budget_ns);
                mbar_wait(&bar[V_FULL + j % C::stages], ph, a.wait_budget_ns);
            }
        }
    } else if (warp == 5) {
        // ---------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc_s = umma_idesc_bf16(kTok, N, 0, 0);   // K (K-major) . Q^T (K-major)
            const uint32_t idesc_o = umma_idesc_bf16(kD, N, 1, 1);     // V^T (MN-major) . P^T (MN-major)
            const uint32_t q_addr = smem_u32(qs);
            const uint32_t p_addr = smem_u32(ps);
            bool ok = true;
            int pv_done = 0;
            for (int j = 0; ok && j <= ntiles; ++j) {
                if (j < ntiles) {
                    const int s = j % C::stages;
                    if (!wait_or_fail(&bar[K_FULL + s], (j / C::stages) & 1, a, err)) { ok = false; break; }
                    if (j >= 2 && !wait_or_fail(&bar[S_FREE + (j & 1)], ((j >> 1) - 1) & 1, a, err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t k_addr = smem_u32(smem + s * C::stage_bytes);
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks) {
                        const uint32_t ka = k_addr + (ks >> 2) * kHalf + (ks & 3) * 32;
                        const uint32_t qa = q_addr + (ks >> 2) * C::q_half + (ks & 3) * 32;
                        umma_bf16_ss(tS[j & 1], umma_smem_desc(ka, 16, 1024, 2), umma_smem_desc(qa, 16, 1024, 2),
                                     idesc_s, ks > 0 ? 1u : 0u);
                    }
                    umma_commit(&bar[S_FULL + (j & 1)]);
                }
                if (j >= 1) {
                    const int jp = j - 1;
                    const int s = jp % C::stages;
                    if (!wait_or_fail(&bar[P_FULL], jp & 1, a, err)) { ok = false; break; }
                    if (!wait_or_fail(&bar[V_FULL + s], (jp / C::stages) & 1, a, err)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t v_addr = smem_u32(smem + s * C::stage_bytes + kTile);
                    // O^T += V^T P_hi^T + V^T P_lo^T: the weights carried as a sum of two bf16 terms
#pragma unroll
                    for (int part = 0; part < 2; ++part) {
#pragma unroll
                        for (int ks = 0; ks < kTok / 16; ++ks) {
                            // A = V^T: 16 tokens (two 8-row groups, 1024 B apart), 64-column blocks kHalf apart
                            // B = P^T: 16 tokens (two 128-byte core-matrix groups), 8-head blocks 2048 B apart
                            umma_bf16_ss(tO, umma_smem_desc(v_addr + ks * 2048, kHalf, 1024, 2),
                                         umma_smem_desc(p_addr + part * C::p_bytes + ks * 256, 128, 2048, 0),
                                         idesc_o, (jp > 0 || part > 0 || ks > 0) ? 1u : 0u);
                        }
                    }
                    umma_commit(&bar[P_FREE]);
                    umma_commit(&bar[KV_EMPTY + s]);
                    ++pv_done;
                }
            }
            if (ok && pv_done == ntiles) umma_commit(&bar[O_FULL]);
            umma_commit(&bar[DRAIN]);
            mbar_wait(&bar[DRAIN], 0, a.wait_budget_ns);
        }
    } else {
        // ---------------- softmax: thread t owns token t of each tile (and d = t of O^T)
        const int t = threadIdx.x;                 // warps 0..3: TMEM lane quarter = warp
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        float m_use[N], l_part[N];
#pragma unroll
        for (int h = 0; h < N; ++h) {
            m_use[h] = -INFINITY;
            l_part[h] = 0.f;
        }
        bool ok = true;
        int uses = 0;
        for (int j = 0; j < ntiles; ++j) {
            const int sb = j & 1;
            if (!wait_or_fail(&bar[S_FULL + sb], (j >> 1) & 1, a, err)) { ok = false; break; }
            tc_fence_after();
            uint32_t raw[N];
            tmem_ld_row<N>(tS[sb] + lane_off, raw);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&bar[S_FREE + sb]);

            const bool valid = (t_begin + j * kTok + t) < t_end;
            float x[N];
            bool over = false;
#pragma unroll
            for (int h = 0; h < N; ++h) {
                x[h] = valid ? __uint_as_float(raw[h]) * a.qscale : -INFINITY;
                over |= x[h] > m_use[h] + kMoveThreshold;
            }
            const int wflag = __any_sync(0xffffffffu, over) ? 1 : 0;
            if (lane == 0) vote[sb * 4 + warp] = wflag;
            if (!group_sync(&bar[GRP], uses, a, err)) { ok = false; break; }
            const bool any_move = (vote[sb * 4 + 0] | vote[sb * 4 + 1] | vote[sb * 4 + 2] | vote[sb * 4 + 3]) != 0;
            float alpha[N];
            bool rescale_o = false;
#pragma unroll
            for (int h = 0; h < N; ++h) alpha[h] = 1.f;
            if (any_move) {
                // CTA-wide maximum of this tile, per head
#pragma unroll
                for (int h = 0; h < N; ++h) {
                    float mx = x[h];
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                    if (lane == 0) red[(sb * 4 + warp) * N + h] = mx;
                }
                if (!group_sync(&bar[GRP], uses, a, err)) { ok = false; break; }
#pragma unroll
                for (int h = 0; h < N; ++h) {
                    const float* rr = red + sb * 4 * N + h;
                    const float tm = fmaxf(fmaxf(rr[0], rr[N]), fmaxf(rr[2 * N], rr[3 * N]));
                    const float m_new = fmaxf(m_use[h], tm);
                    if (m_new > m_use[h] + kMoveThreshold) {
                        alpha[h] = ex2(m_use[h] - m_new);     // 0 on the first tile
                        m_use[h] = m_new;
                        l_part[h] *= alpha[h];
                        rescale_o = true;
                    }
                }
                rescale_o = rescale_o && (j > 0);             // uniform: every thread saw the same maxima
            }
            float p[N];
#pragma unroll
            for (int h = 0; h < N; ++h) {
                p[h] = ex2(x[h] - m_use[h]);
                l_part[h] += p[h];
            }
            if (j >= 1) {
                if (!wait_or_fail(&bar[P_FREE], (j - 1) & 1, a, err)) { ok = false; break; }
                tc_fence_after();
                if (rescale_o) {
                    uint32_t o[N];
                    tmem_ld_row<N>(tO + lane_off, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int h = 0; h < N; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
                    tmem_st_row<N>(tO + lane_off, o);
                    tmem_wait_st();
                }
            }
            // Rows past the history may hold anything (NaN included) and the tensor cores would form
            // 0 * NaN: in a partial tile the masked tokens zero their own V row once it has landed.
            if (t_end - (t_begin + j * kTok) < kTok) {
                const int st = j % C::stages;
                if (!valid) {
                    if (!wait_or_fail(&bar[V_FULL + st], (j / C::stages) & 1, a, err)) { ok = false; break; }
                    uint8_t *vrow = smem + st * C::stage_bytes + kTile + t * 128;
                    const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        *reinterpret_cast<uint4 *>(vrow + c * 16) = z;
                        *reinterpret_cast<uint4 *>(vrow + kHalf + c * 16) = z;
                    }
                }
            }
            // P^T, MN-major without swizzle: core matrices of 8 tokens x 8 heads (128 B).  Each weight is
            // stored as hi = bf16(p) plus lo = bf16(p - hi), so the PV product sees p to about 2^-17.
#pragma unroll
            for (int hb = 0; hb < N / 8; ++hb) {
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float a0 = p[hb * 8 + 2 * e], a1 = p[hb * 8 + 2 * e + 1];
                    hi[e] = pack2(a0, a1);
                    lo[e] = pack2(a0 - bf16_lo(hi[e]), a1 - bf16_hi(hi[e]));
                }
                uint8_t *dst = ps + hb * 2048 + (t >> 3) * 128 + (t & 7) * 16;
                *reinterpret_cast<uint4 *>(dst) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4 *>(dst + C::p_bytes) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bar[P_FULL]);
        }
        // sums of the weights per head over the CTA's tokens
        if (ok) {
#pragma unroll
            for (int h = 0; h < N; ++h) {
                float v = l_part[h];
                v += __shfl_xor_sync(0xffffffffu, v, 16);
                v += __shfl_xor_sync(0xffffffffu, v, 8);
                v += __shfl_xor_sync(0xffffffffu, v, 4);
                v += __shfl_xor_sync(0xffffffffu, v, 2);
                v += __shfl_xor_sync(0xffffffffu, v, 1);
                if (lane == 0) lsum[warp * N + h] = v;
            }
            ok = group_sync(&bar[GRP], uses, a, err);
        }
        if (ok && wait_or_fail(&bar[O_FULL], 0, a, err)) {
            tc_fence_after();
            uint32_t o[N];
            tmem_ld_row<N>(tO + lane_off, o);
            tmem_wait_ld();
            const int d = t;
#pragma unroll
            for (int h = 0; h < N; ++h) {
                if (h >= g) break;
                const float L = lsum[h] + lsum[N + h] + lsum[2 * N + h] + lsum[3 * N + h];
                const float O = __uint_as_float(o[h]);
                const size_t row = (size_t)b * a.Hq + h0 + h;
                if (a.nsplit == 1) {
                    a.out[row * kD + d] = __float2bfloat16_rn(L > 0.f ? O / L : 0.f);
                } else {
                    const size_t prow = row * a.nsplit + split;
                    a.part_o[prow * kD + d] = O;
                    if (d == 0) {
                        a.part_ml[prow * 2 + 0] = m_use[h];
                        a.part_ml[prow * 2 + 1] = L;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, C::tmem_cols);
    }
}

template <int N>
cudaError_t launch_tc(const CUtensorMap &tmK, const CUtensorMap &tmV, const DecodeArgs &a, cudaStream_t stream)
{
    const int smem = TcCfg<N>::bytes + 1024;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel<N>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        attr_done[dev] = true;
    }
    dim3 grid(a.nsplit, a.Hkv, a.B);
    decode_tc_kernel<N><<<grid, kThreads, smem, stream>>>(tmK, tmV, a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_tc(const CUtensorMap &tmK, const CUtensorMap &tmV, const DecodeArgs &a,
                             cudaStream_t stream)
{
    if (a.group <= 16) return launch_tc<16>(tmK, tmV, a, stream);
    if (a.group <= 32) return launch_tc<32>(tmK, tmV, a, stream);
    return cudaErrorInvalidValue;
}

}  // namespace gqa
