// mla.cu -- MLA decode with absorbed weights on the CUDA cores (a first, plain path).
//
// The operator ("MLA: multi-head latent attention", anrans.github.io attention-variants):
// out[b,h] = sum_{t < seqlens[b]} softmax_t(scale * q[b,h] . kv[b,t]) kv[b,t,0:512], where a
// cached row kv[b,t] is the 512-wide latent followed by the 64-wide RoPE key shared by all
// heads, and q[b,h] is the head's absorbed latent query followed by its RoPE query.
//
// One CTA takes 16 query heads of one sequence over one token range (split-KV); tiles of 32
// cached rows go through shared memory once for those 16 heads.  Per tile: the scores (each warp
// takes four tokens, its lanes split the 576 coordinates and shuffle-reduce the 16 heads' dot
// products), a base-2 online softmax per head (one warp per two heads, one lane per token), then
// the weighted latent rows added into per-thread fp32 accumulators (thread = one head x 32 latent
// coordinates).  Ranges of one sequence are merged by mla_combine_kernel (log-sum-exp).
//
// The work is a dense contraction (2 x Hq x (576 + 512) FLOP per cached token, about 242 FLOP per
// byte at 128 heads), which belongs on the tensor cores; this kernel is the correct baseline that
// the tensor-core version is checked and measured against.
#include "mla.h"

#include <algorithm>

#include "ptx.cuh"

namespace gqa {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kOut = 32;                                // latent coordinates per thread in the PV step
constexpr int kRowChunks = kMlaRow * 2 / 16;            // 16-byte chunks per cached row (72)
constexpr size_t kQsBytes = sizeof(float) * kMlaHeads * kMlaRow;
constexpr size_t kKvBytes = sizeof(__nv_bfloat16) * kMlaTile * kMlaRow;
constexpr size_t kPsBytes = sizeof(float) * kMlaHeads * kMlaTile;
constexpr size_t kSmemBytes = kQsBytes + kKvBytes + kPsBytes + 3 * sizeof(float) * kMlaHeads;
static_assert(kMlaHeads * 16 == kThreads, "PV step: 16 threads per head");
static_assert(kOut * 16 == kMlaLatent, "PV step: 16 threads cover the latent");
static_assert(kMlaHeads == 2 * kWarps, "softmax step: two heads per warp");
static_assert(kMlaTile == 32, "softmax step: one lane per token");
static_assert(kQsBytes % 16 == 0 && kKvBytes % 16 == 0, "16-byte aligned shared-memory regions");

__global__ void __launch_bounds__(kThreads) mla_decode_kernel(const MlaArgs a)
{
    extern __shared__ __align__(16) unsigned char smem[];
    float *qs = reinterpret_cast<float *>(smem);                                    // [16][576]
    __nv_bfloat16 *kvs = reinterpret_cast<__nv_bfloat16 *>(smem + kQsBytes);        // [32][576]
    float *ps = reinterpret_cast<float *>(smem + kQsBytes + kKvBytes);              // [16][32]
    float *ms = ps + kMlaHeads * kMlaTile;                                          // running max
    float *ls = ms + kMlaHeads;                                                     // weight sum
    float *al = ls + kMlaHeads;                                                     // tile rescale

    const int split = blockIdx.x, b = blockIdx.z;
    const int h0 = blockIdx.y * kMlaHeads;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int T = min(max(a.seqlens[b], 0), a.Tmax);
    const int t_begin = split * a.chunk;
    const int t_end = min(t_begin + a.chunk, T);

    // the block's query rows times scale * log2(e), in fp32; heads past Hq are zero rows
    for (int i = tid; i < kMlaHeads * kMlaRow; i += kThreads) {
        const int h = h0 + i / kMlaRow;
        qs[i] = h < a.Hq ? __bfloat162float(a.q[((size_t)b * a.Hq + h) * kMlaRow + i % kMlaRow]) * a.qscale : 0.f;
    }
    if (tid < kMlaHeads) {
        ms[tid] = -INFINITY;
        ls[tid] = 0.f;
        al[tid] = 1.f;
    }
    // PV ownership: head ph, latent coordinates pd + 128 c + e (c < 4, e < 8): the 16 threads of a
    // head read consecutive 16-byte pieces of a row
    const int ph = tid >> 4;
    const int pd = (tid & 15) * 8;
    float o[kOut];
#pragma unroll
    for (int i = 0; i < kOut; ++i) o[i] = 0.f;
    __syncthreads();

    for (int t0 = t_begin; t0 < t_end; t0 += kMlaTile) {
        const int n = min(kMlaTile, t_end - t0);
        // 1. the tile's cached rows; rows past the range are zeros, never read from the cache
        const uint4 *src = reinterpret_cast<const uint4 *>(a.kv + ((size_t)b * a.Tmax + t0) * kMlaRow);
        uint4 *dst = reinterpret_cast<uint4 *>(kvs);
        for (int i = tid; i < kMlaTile * kRowChunks; i += kThreads)
            dst[i] = (i / kRowChunks) < n ? src[i] : make_uint4(0u, 0u, 0u, 0u);
        __syncthreads();

        // 2. scores in log2 units: warp w takes tokens w, w + 8, w + 16, w + 24
        for (int j = warp; j < kMlaTile; j += kWarps) {
            float acc[kMlaHeads];
#pragma unroll
            for (int hh = 0; hh < kMlaHeads; ++hh) acc[hh] = 0.f;
            if (j < n) {
                for (int k = lane; k < kMlaRow; k += 32) {
                    const float x = __bfloat162float(kvs[j * kMlaRow + k]);
#pragma unroll
                    for (int hh = 0; hh < kMlaHeads; ++hh) acc[hh] = fmaf(qs[hh * kMlaRow + k], x, acc[hh]);
                }
            }
#pragma unroll
            for (int hh = 0; hh < kMlaHeads; ++hh) {
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) acc[hh] += __shfl_xor_sync(0xffffffffu, acc[hh], off);
            }
            if (lane == 0) {
#pragma unroll
                for (int hh = 0; hh < kMlaHeads; ++hh) ps[hh * kMlaTile + j] = j < n ? acc[hh] : -INFINITY;
            }
        }
        __syncthreads();

        // 3. online softmax: warp w takes heads 2w and 2w + 1, lane = token
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int hh = warp * 2 + e;
            const float x = lane < n ? ps[hh * kMlaTile + lane] : -INFINITY;
            float mt = x;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
            const float m_old = ms[hh];
            const float m_new = fmaxf(m_old, mt);
            const float alpha = (m_old == -INFINITY) ? 0.f : ex2(m_old - m_new);
            const float p = lane < n ? ex2(x - m_new) : 0.f;
            float sum = p;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
            ps[hh * kMlaTile + lane] = p;
            __syncwarp();
            if (lane == 0) {
                ls[hh] = ls[hh] * alpha + sum;
                ms[hh] = m_new;
                al[hh] = alpha;
            }
        }
        __syncthreads();

        // 4. o = alpha o + sum_j p_j latent_j for this thread's head and coordinates
        const float alpha = al[ph];
#pragma unroll
        for (int i = 0; i < kOut; ++i) o[i] *= alpha;
        for (int j = 0; j < n; ++j) {
            const float p = ps[ph * kMlaTile + j];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint4 v = *reinterpret_cast<const uint4 *>(kvs + j * kMlaRow + pd + 128 * c);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    o[c * 8 + 2 * e] = fmaf(p, __uint_as_float(w[e] << 16), o[c * 8 + 2 * e]);
                    o[c * 8 + 2 * e + 1] = fmaf(p, __uint_as_float(w[e] & 0xffff0000u), o[c * 8 + 2 * e + 1]);
                }
            }
        }
        __syncthreads();   // the next tile overwrites kvs and ps
    }

    const int h = h0 + ph;
    if (h >= a.Hq) return;
    const float l = ls[ph];
    const size_t row = (size_t)b * a.Hq + h;
    if (a.nsplit == 1) {
        // a zero sum only for an empty history (output 0); a NaN sum (a NaN in the cache) stays NaN
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int e = 0; e < 8; ++e)
                a.out[row * kMlaLatent + pd + 128 * c + e] = __float2bfloat16_rn(l != 0.f ? o[c * 8 + e] / l : 0.f);
    } else {
        const size_t prow = row * a.nsplit + split;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int e = 0; e < 8; ++e) a.part_o[prow * kMlaLatent + pd + 128 * c + e] = o[c * 8 + e];
        if ((tid & 15) == 0) {
            a.part_ml[prow * 2 + 0] = ms[ph];
            a.part_ml[prow * 2 + 1] = l;
        }
    }
}

// One CTA per (head, sequence), four latent coordinates per thread: the ranges' partials merged
// with weights 2^(m_s - M), M their largest maximum (empty ranges carry m = -inf and weigh 0).
__global__ void __launch_bounds__(kMlaLatent / 4) mla_combine_kernel(const MlaArgs a)
{
    const int h = blockIdx.x, b = blockIdx.y;
    const int d = threadIdx.x * 4;
    const size_t row = (size_t)b * a.Hq + h;
    const float *ml = a.part_ml + row * a.nsplit * 2;
    float M = -INFINITY;
    for (int s = 0; s < a.nsplit; ++s) M = fmaxf(M, ml[2 * s]);
    float L = 0.f, O[4] = {0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < a.nsplit; ++s) {
        const float m = ml[2 * s];
        const float w = (m == -INFINITY) ? 0.f : ex2(m - M);
        L += ml[2 * s + 1] * w;
        const float4 p = *reinterpret_cast<const float4 *>(a.part_o + (row * a.nsplit + s) * kMlaLatent + d);
        O[0] += p.x * w;
        O[1] += p.y * w;
        O[2] += p.z * w;
        O[3] += p.w * w;
    }
    // a zero sum only for an empty history (output 0); a NaN sum (a NaN in the cache) stays NaN
#pragma unroll
    for (int i = 0; i < 4; ++i) a.out[row * kMlaLatent + d + i] = __float2bfloat16_rn(L != 0.f ? O[i] / L : 0.f);
}

}  // namespace

MlaPlan mla_plan_host(int B, int Hq, int Tmax, int num_sms)
{
    // about two CTAs per SM over (range, head block, sequence), ranges of at least 256 tokens
    const long long blocks = (long long)B * ((Hq + kMlaHeads - 1) / kMlaHeads);
    const long long want = (2LL * num_sms + blocks - 1) / blocks;
    int nsplit = (int)std::max(1LL, std::min(want, (long long)(Tmax + 255) / 256));
    int chunk = (Tmax + nsplit - 1) / nsplit;
    chunk = (chunk + kMlaTile - 1) / kMlaTile * kMlaTile;
    nsplit = (Tmax + chunk - 1) / chunk;
    MlaPlan p;
    p.nsplit = nsplit;
    p.chunk = chunk;
    p.ws_bytes = nsplit > 1 ? (size_t)B * Hq * nsplit * (kMlaLatent + 2) * sizeof(float) : 0;
    return p;
}

cudaError_t launch_mla_decode(const MlaArgs &a, cudaStream_t stream, int *launches, cudaEvent_t before,
                              cudaEvent_t after)
{
    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
        const cudaError_t e =
            cudaFuncSetAttribute(mla_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_done[dev] = true;
    }
    const dim3 grid(a.nsplit, (a.Hq + kMlaHeads - 1) / kMlaHeads, a.B);
    if (before) cudaEventRecord(before, stream);
    mla_decode_kernel<<<grid, kThreads, kSmemBytes, stream>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (after) cudaEventRecord(after, stream);
    ++*launches;
    if (a.nsplit > 1) {
        mla_combine_kernel<<<dim3(a.Hq, a.B), kMlaLatent / 4, 0, stream>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        ++*launches;
    }
    return cudaSuccess;
}

}  // namespace gqa
