// decode.cu -- GQA single-token decode over a bf16 KV cache (split-KV).
//
// One CTA serves one (sequence b, KV head, KV split) tile and, inside it, a
// block of up to HB query heads of that KV head's group.  A producer warp
// streams the split's K/V rows through a ring of shared-memory stages with
// TMA; each stage is fetched from HBM once and read by every query head of
// the block ("Kernels do not need to copy the KV heads", anrans.github.io
// attention-variants: a group's query heads are extra query rows against one
// shared KV head).  Consumer warps do the dot products with packed fp32 FMAs
// and keep a running maximum / sum per head (online softmax in base 2, the
// scale folded into q together with log2 e); the CTA merges its warps and
// either writes the bf16 output or one split's partial result, which
// decode_combine_kernel merges with a log-sum-exp reduction.
//
// Shared-memory stage layout: K and V tiles of kDecodeTile tokens, each split
// into two 64-column halves written by TMA with the 128-byte swizzle (row r,
// 16-byte chunk c lands at chunk c ^ (r & 7)), so that both the
// one-token-per-lane reads of the score phase and the one-row-per-warp reads
// of the value phase are free of bank conflicts.
#include "internal.h"
#include "ptx.cuh"

namespace gqa {

namespace {

constexpr int kD = kHeadDim;
constexpr int kHalf = 64;                 // bf16 elements per 128-byte swizzled row
constexpr int kNW = 4;                    // consumer warps
constexpr int kTPW = kDecodeTile / kNW;   // tokens per consumer warp per stage (16)
constexpr int kTT = kDecodeTile;          // tokens per stage
constexpr int kStages = 3;
constexpr int kQPitch = kHalf + 4;        // floats per (head, half) row of the fp32 query copy
constexpr int kHalfBytes = kTT * 128;     // one 64-column half of one K or V tile
constexpr int kStageBytes = 4 * kHalfBytes;
constexpr int kThreads = (kNW + 1) * 32;

static_assert(kTPW == 16, "score phase maps 16 tokens onto the 16 lane pairs of a warp");

template <int HB>
struct SmemLayout {
    static constexpr int q_off = kStages * kStageBytes;
    static constexpr int p_off = q_off + HB * 2 * kQPitch * 4;
    static constexpr int bar_off = p_off + kNW * kTPW * HB * 4;
    static constexpr int err_off = bar_off + 2 * kStages * 8;
    static constexpr int bytes = err_off + 16;
    // merge scratch reuses the stage ring once every tile is consumed
    static_assert(kNW * HB * (kD + 2) * 4 <= kStages * kStageBytes, "merge scratch must fit the stage ring");
};

__device__ __forceinline__ void record_status(int *status, int code)
{
    if (status) atomicCAS(status, 0, code);
}

template <int HB>
__global__ void __launch_bounds__(kThreads, kDecodeCtasPerSm)
decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const DecodeArgs a)
{
    using L = SmemLayout<HB>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int split = blockIdx.x;
    const int kvh = blockIdx.y / a.nhb;
    const int hb = blockIdx.y % a.nhb;
    const int b = blockIdx.z;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    int T = a.seqlens[b];
    T = T < 0 ? 0 : (T > a.Tmax ? a.Tmax : T);
    const int t_begin = split * a.chunk;
    const int t_end = min(t_begin + a.chunk, T);
    const int h0 = kvh * a.group + hb * HB;          // first query head of this CTA
    const int nh = min(HB, a.group - hb * HB);       // query heads handled here

    if (t_end <= t_begin) {
        // nothing cached in this split; with a single split the output row is zero
        if (a.nsplit == 1) {
            uint4 z = make_uint4(0, 0, 0, 0);
            for (int i = threadIdx.x; i < nh * (kD / 8); i += kThreads) {
                const int hh = i / (kD / 8), c = i % (kD / 8);
                reinterpret_cast<uint4 *>(a.out + ((size_t)b * a.Hq + h0 + hh) * kD)[c] = z;
            }
        }
        return;
    }
    const int ntiles = (t_end - t_begin + kTT - 1) / kTT;

    float *q_s = reinterpret_cast<float *>(smem + L::q_off);
    float *p_s = reinterpret_cast<float *>(smem + L::p_off);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::bar_off);
    uint64_t *empty = full + kStages;
    volatile int *err = reinterpret_cast<volatile int *>(smem + L::err_off);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kNW);
        }
        *err = 0;
        fence_barrier_init();
    }
    // the block's query rows, pre-multiplied by scale * log2(e), as fp32 [head][half][kQPitch]
    for (int i = threadIdx.x; i < HB * kD; i += kThreads) {
        const int hh = i / kD, j = i % kD;
        float x = 0.f;
        if (hh < nh) x = __bfloat162float(a.q[((size_t)b * a.Hq + h0 + hh) * kD + j]) * a.qscale;
        q_s[(hh * 2 + j / kHalf) * kQPitch + (j % kHalf)] = x;
    }
    __syncthreads();

    if (warp == kNW) {
        // ---------------- producer: one elected lane issues the TMA loads
        if (lane == 0) {
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            int issued = 0;
            for (int it = 0; it < ntiles; ++it) {
                const int s = it % kStages;
                const uint32_t ph = (it / kStages) & 1;
                if (*err || !mbar_wait(&empty[s], ph ^ 1, a.wait_budget_ns)) {
                    *err = 1;
                    record_status(a.status, kStatusTimeout);
                    break;
                }
                uint8_t *st = smem + s * kStageBytes;
                const int t0 = t_begin + it * kTT;
                mbar_arrive_expect_tx(&full[s], kStageBytes);
                tma_load_4d(st + 0 * kHalfBytes, &tmK, &full[s], 0, kvh, t0, b);
                tma_load_4d(st + 1 * kHalfBytes, &tmK, &full[s], kHalf, kvh, t0, b);
                tma_load_4d(st + 2 * kHalfBytes, &tmV, &full[s], 0, kvh, t0, b);
                tma_load_4d(st + 3 * kHalfBytes, &tmV, &full[s], kHalf, kvh, t0, b);
                ++issued;
            }
            // never leave with copies in flight: wait (bounded) for the last loads of each stage
            for (int it = issued - 1; it >= 0 && it >= issued - kStages; --it) {
                if (!mbar_wait(&full[it % kStages], (it / kStages) & 1, a.wait_budget_ns)) {
                    record_status(a.status, kStatusTimeout);
                    break;
                }
            }
        }
        return;
    }

    // ---------------- consumers
    const int t16 = lane & 15;     // token of this lane pair in the warp's 16-token slice
    const int half = lane >> 4;    // score phase: which 64-column half of d this lane sums
    const int pv_chunk = (lane & 15) >> 1;  // value phase: 16-byte chunk within the half row
    const int pv_sub = lane & 1;            // value phase: 8-byte half of that chunk
    float *pw = p_s + warp * kTPW * HB;

    float m[HB], l[HB];
    float2 o[HB][2];  // this lane's 4 output columns: d = 64*half + 8*pv_chunk + 4*pv_sub + 0..3
#pragma unroll
    for (int hh = 0; hh < HB; ++hh) {
        m[hh] = -INFINITY;
        l[hh] = 0.f;
        o[hh][0] = make_float2(0.f, 0.f);
        o[hh][1] = make_float2(0.f, 0.f);
    }

    bool ok = true;
    for (int it = 0; it < ntiles; ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (!mbar_wait(&full[s], ph, a.wait_budget_ns)) {
            *err = 1;
            record_status(a.status, kStatusTimeout);
            ok = false;
            break;
        }
        const uint8_t *st = smem + s * kStageBytes;
        const int slice0 = t_begin + it * kTT + warp * kTPW;   // first token of this warp's slice
        int nvalid = t_end - slice0;
        nvalid = nvalid < 0 ? 0 : (nvalid > kTPW ? kTPW : nvalid);

        // ---- scores: lane pair (t16, half) sums its half of q.k for token slice0 + t16
        const int r = warp * kTPW + t16;                // row within the stage
        const uint8_t *krow = st + half * kHalfBytes + r * 128;
        float2 acc[HB];
#pragma unroll
        for (int hh = 0; hh < HB; ++hh) acc[hh] = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const uint4 kr = *reinterpret_cast<const uint4 *>(krow + ((c ^ (r & 7)) << 4));
            const float2 k01 = make_float2(bf16_lo(kr.x), bf16_hi(kr.x));
            const float2 k23 = make_float2(bf16_lo(kr.y), bf16_hi(kr.y));
            const float2 k45 = make_float2(bf16_lo(kr.z), bf16_hi(kr.z));
            const float2 k67 = make_float2(bf16_lo(kr.w), bf16_hi(kr.w));
#pragma unroll
            for (int hh = 0; hh < HB; ++hh) {
                const float *qp = q_s + (hh * 2 + half) * kQPitch + c * 8;
                const float4 qa = *reinterpret_cast<const float4 *>(qp);
                const float4 qb = *reinterpret_cast<const float4 *>(qp + 4);
                acc[hh] = __ffma2_rn(k01, make_float2(qa.x, qa.y), acc[hh]);
                acc[hh] = __ffma2_rn(k23, make_float2(qa.z, qa.w), acc[hh]);
                acc[hh] = __ffma2_rn(k45, make_float2(qb.x, qb.y), acc[hh]);
                acc[hh] = __ffma2_rn(k67, make_float2(qb.z, qb.w), acc[hh]);
            }
        }
        // ---- online softmax over the slice (base 2), per head
        float alpha[HB];
#pragma unroll
        for (int hh = 0; hh < HB; ++hh) {
            float x = acc[hh].x + acc[hh].y;
            x += __shfl_xor_sync(0xffffffffu, x, 16);
            x = (t16 < nvalid) ? x : -INFINITY;
            float mx = x;
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            const float mnew = fmaxf(m[hh], mx);
            float p = 0.f;
            alpha[hh] = 1.f;
            if (mnew != -INFINITY) {
                alpha[hh] = ex2(m[hh] - mnew);
                p = ex2(x - mnew);
            }
            m[hh] = mnew;
            l[hh] = l[hh] * alpha[hh] + (half == 0 ? p : 0.f);
            if (half == 0) pw[t16 * HB + hh] = p;
        }
        __syncwarp();

        // ---- values: o = alpha * o + sum_t p_t v_t over the slice's valid tokens
#pragma unroll
        for (int hh = 0; hh < HB; ++hh) {
            const float2 al = make_float2(alpha[hh], alpha[hh]);
            o[hh][0] = __fmul2_rn(o[hh][0], al);
            o[hh][1] = __fmul2_rn(o[hh][1], al);
        }
        const uint8_t *vbase = st + 2 * kHalfBytes + half * kHalfBytes + pv_sub * 8;
        for (int t = 0; t < nvalid; ++t) {
            const int rr = warp * kTPW + t;
            const uint2 vr = *reinterpret_cast<const uint2 *>(vbase + rr * 128 + ((pv_chunk ^ (rr & 7)) << 4));
            const float2 v01 = make_float2(bf16_lo(vr.x), bf16_hi(vr.x));
            const float2 v23 = make_float2(bf16_lo(vr.y), bf16_hi(vr.y));
            const float *pt = pw + t * HB;
#pragma unroll
            for (int hh = 0; hh < HB; ++hh) {
                const float2 pp = make_float2(pt[hh], pt[hh]);
                o[hh][0] = __ffma2_rn(pp, v01, o[hh][0]);
                o[hh][1] = __ffma2_rn(pp, v23, o[hh][1]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }

    // every consumer warp must be past its last stage before the ring is reused as scratch
    named_barrier_sync(1, kNW * 32);
    if (!ok || *err) return;

#pragma unroll
    for (int hh = 0; hh < HB; ++hh) {
        float x = l[hh];
        x += __shfl_xor_sync(0xffffffffu, x, 16);
        x += __shfl_xor_sync(0xffffffffu, x, 8);
        x += __shfl_xor_sync(0xffffffffu, x, 4);
        x += __shfl_xor_sync(0xffffffffu, x, 2);
        x += __shfl_xor_sync(0xffffffffu, x, 1);
        l[hh] = x;
    }
    float *mo = reinterpret_cast<float *>(smem);        // [kNW][HB][kD]
    float *mm = mo + kNW * HB * kD;                     // [kNW][HB]
    float *ml = mm + kNW * HB;                          // [kNW][HB]
    const int dcol = half * kHalf + pv_chunk * 8 + pv_sub * 4;
#pragma unroll
    for (int hh = 0; hh < HB; ++hh) {
        *reinterpret_cast<float4 *>(mo + (warp * HB + hh) * kD + dcol) =
            make_float4(o[hh][0].x, o[hh][0].y, o[hh][1].x, o[hh][1].y);
        if (lane == 0) {
            mm[warp * HB + hh] = m[hh];
            ml[warp * HB + hh] = l[hh];
        }
    }
    named_barrier_sync(1, kNW * 32);

    for (int i = threadIdx.x; i < nh * kD; i += kNW * 32) {
        const int hh = i / kD, j = i % kD;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kNW; ++w) M = fmaxf(M, mm[w * HB + hh]);
        float Lsum = 0.f, O = 0.f;
#pragma unroll
        for (int w = 0; w < kNW; ++w) {
            const float mw = mm[w * HB + hh];
            const float f = (mw == -INFINITY) ? 0.f : ex2(mw - M);
            Lsum += ml[w * HB + hh] * f;
            O += mo[(w * HB + hh) * kD + j] * f;
        }
        const size_t row = (size_t)b * a.Hq + h0 + hh;
        if (a.nsplit == 1) {
            // a zero sum only for an empty history (output 0); a NaN sum (a NaN in the cache) stays NaN
            a.out[row * kD + j] = __float2bfloat16_rn(Lsum != 0.f ? O / Lsum : 0.f);
        } else {
            const size_t prow = row * a.nsplit + split;
            a.part_o[prow * kD + j] = O;
            if (j == 0) {
                a.part_ml[prow * 2 + 0] = M;
                a.part_ml[prow * 2 + 1] = Lsum;
            }
        }
    }
}

// Merge the split partials of one (b, query head):
// out = sum_s o_s 2^(m_s-M) / sum_s l_s 2^(m_s-M), M = max_s m_s.  The (m, l) pairs are read by all
// threads at once (one split per thread), the maximum and the weights go through shared memory, and
// the weighted sum over o_s is unrolled so that its loads are in flight together.
__global__ void __launch_bounds__(kD) decode_combine_kernel(const DecodeArgs a)
{
    // launched as a programmatic dependent of the split kernel: wait for its results
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int h = blockIdx.x, b = blockIdx.y, j = threadIdx.x;
    const size_t row = (size_t)b * a.Hq + h;
    const float2 *ml = reinterpret_cast<const float2 *>(a.part_ml) + row * a.nsplit;
    const float *po = a.part_o + row * a.nsplit * kD + j;
    // The first kSpec slots are fetched together with the piece count, so that one round trip serves
    // every history of up to kSpec pieces; slots past the count are never used (they may hold anything).
    constexpr int kSpec = 8;
    float2 mlv[kSpec];
    float ov[kSpec];
    int nv;
    if (a.nsplit_b) {
        nv = a.nsplit_b[b];
    } else {
        int T = a.seqlens[b];
        T = T < 0 ? 0 : (T > a.Tmax ? a.Tmax : T);
        nv = (T + a.chunk - 1) / a.chunk;
    }
#pragma unroll
    for (int s = 0; s < kSpec; ++s) {
        if (s < a.nsplit) {
            mlv[s] = ml[s];
            ov[s] = po[(size_t)s * kD];
        } else {
            mlv[s] = make_float2(-INFINITY, 0.f);
            ov[s] = 0.f;
        }
    }
    // with the device plan, a history of one piece (or none) was written out by the split kernel
    if (a.nsplit_b && nv <= 1) return;
    nv = nv > a.nsplit ? a.nsplit : nv;
    // M = max over the pieces
    float M = -INFINITY;
#pragma unroll
    for (int s = 0; s < kSpec; ++s)
        if (s < nv) M = fmaxf(M, mlv[s].x);
    for (int s = kSpec; s < nv; ++s) M = fmaxf(M, ml[s].x);
    float Lsum = 0.f, O = 0.f;
#pragma unroll
    for (int s = 0; s < kSpec; ++s) {
        if (s < nv) {
            const float wgt = ex2(mlv[s].x - M);
            O += ov[s] * wgt;
            Lsum += mlv[s].y * wgt;
        }
    }
    for (int s = kSpec; s < nv; s += 4) {
        float2 m4[4];
        float o4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (s + e < nv) {
                m4[e] = ml[s + e];
                o4[e] = po[(size_t)(s + e) * kD];
            }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (s + e < nv) {
                const float wgt = ex2(m4[e].x - M);
                O += o4[e] * wgt;
                Lsum += m4[e].y * wgt;
            }
        }
    }
    // a zero sum only for an empty history (output 0); a NaN sum (a NaN in the cache) stays NaN
    a.out[row * kD + j] = __float2bfloat16_rn(Lsum != 0.f ? O / Lsum : 0.f);
}

// The deliberately expanded baseline: physically repeat each KV head for its g
// query heads (rows t < seqlens[b] only), 16 bytes per thread.
__global__ void repeat_kv_kernel(const uint4 *__restrict__ k, const uint4 *__restrict__ v,
                                 const int32_t *__restrict__ seqlens, uint4 *__restrict__ k_rep,
                                 uint4 *__restrict__ v_rep, int B, int Tmax, int Hq, int Hkv)
{
    const int group = Hq / Hkv;
    const long long total = (long long)B * Tmax * Hq * (kD / 8);
    for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int c = (int)(idx % (kD / 8));
        const long long rowi = idx / (kD / 8);
        const int h = (int)(rowi % Hq);
        const long long bt = rowi / Hq;
        const int t = (int)(bt % Tmax);
        const int b = (int)(bt / Tmax);
        int T = seqlens[b];
        T = T < 0 ? 0 : (T > Tmax ? Tmax : T);
        if (t >= T) continue;
        const long long src = (bt * Hkv + h / group) * (kD / 8) + c;
        k_rep[idx] = k[src];
        v_rep[idx] = v[src];
    }
}

// Waits on a barrier nothing completes, gives up after budget_ns, records a timeout.
__global__ void wait_timeout_selftest_kernel(int *status, unsigned long long budget_ns)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (!mbar_wait(&bar, 0, budget_ns)) record_status(status, kStatusTimeout);
    }
}

template <int HB>
cudaError_t launch_split_hb(const CUtensorMap &tmK, const CUtensorMap &tmV, const DecodeArgs &a,
                            cudaStream_t stream)
{
    const int smem = SmemLayout<HB>::bytes + 1024;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<HB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             smem);
        if (e != cudaSuccess) return e;
        attr_done[dev] = true;
    }
    dim3 grid(a.nsplit, a.Hkv * a.nhb, a.B);
    decode_split_kernel<HB><<<grid, kThreads, smem, stream>>>(tmK, tmV, a);
    return cudaGetLastError();
}

}  // namespace

int decode_heads_per_cta(int g)
{
    if (g <= 1) return 1;
    if (g <= 2) return 2;
    if (g <= 4) return 4;
    return 8;
}

DecodeShape decode_shape(int g)
{
    DecodeShape s;
    s.tensor_cores = (g >= 3 && g <= 32);
    if (s.tensor_cores) {
        s.tile = 128;
        s.heads_per_cta = g;
        s.nhb = 1;
        s.ctas_per_sm = 1;
    } else {
        s.tile = kDecodeTile;
        s.heads_per_cta = decode_heads_per_cta(g);
        s.nhb = (g + s.heads_per_cta - 1) / s.heads_per_cta;
        s.ctas_per_sm = kDecodeCtasPerSm;
    }
    return s;
}

cudaError_t launch_decode_split(const CUtensorMap &tmK, const CUtensorMap &tmV, const DecodeArgs &a,
                                cudaStream_t stream)
{
    switch (decode_heads_per_cta(a.group)) {
    case 1: return launch_split_hb<1>(tmK, tmV, a, stream);
    case 2: return launch_split_hb<2>(tmK, tmV, a, stream);
    case 4: return launch_split_hb<4>(tmK, tmV, a, stream);
    default: return launch_split_hb<8>(tmK, tmV, a, stream);
    }
}

cudaError_t launch_decode_combine(const DecodeArgs &a, cudaStream_t stream, bool pdl)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.Hq, a.B);
    cfg.blockDim = dim3(kD);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, decode_combine_kernel, a);
}

cudaError_t launch_repeat_kv(const void *k, const void *v, const int32_t *seqlens, void *k_rep, void *v_rep,
                             int B, int Tmax, int Hq, int Hkv, cudaStream_t stream)
{
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    repeat_kv_kernel<<<sms * 8, 256, 0, stream>>>(static_cast<const uint4 *>(k), static_cast<const uint4 *>(v),
                                                  seqlens, static_cast<uint4 *>(k_rep),
                                                  static_cast<uint4 *>(v_rep), B, Tmax, Hq, Hkv);
    return cudaGetLastError();
}

cudaError_t launch_wait_timeout_selftest(int *status, unsigned long long budget_ns, cudaStream_t stream)
{
    wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(status, budget_ns);
    return cudaGetLastError();
}

}  // namespace gqa
