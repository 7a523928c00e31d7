// noalloc.cu -- gqa_decode_noalloc: the split-KV decode with its scratch in a
// fixed, file-scope device array instead of memory from cudaMalloc.
//
// Some callers cannot let a library allocate device memory: a serving engine
// that reserves nearly all of the GPU for its own pool (its KV cache) up front
// leaves nothing for a surprise cudaMalloc, and a latency-critical decode loop
// cannot absorb cudaMalloc's implicit synchronisation and unpredictable cost.
// For them this entry point runs the same kernels as gqa_decode with the split
// partials in g_noalloc_scratch, which every GPU that loads this library holds
// for the life of the process.
#include <cudaTypedefs.h>

#include <mutex>

#include "../../include/gqa.h"
#include "internal.h"

namespace {

using namespace gqa;

constexpr size_t kScratchBytes = size_t(32) << 20;   // 32 MiB of split partials per device
static __device__ __align__(256) float g_noalloc_scratch[kScratchBytes / sizeof(float)];

constexpr int kMaxDevices = 64;
std::mutex g_na_mu;
float *g_scratch_addr[kMaxDevices] = {};             // device address of the array, per device
int g_num_sms[kMaxDevices] = {};
PFN_cuTensorMapEncodeTiled_v12000 g_na_encode = nullptr;

// Once per device, with that device current: the array's device address.  In host
// code the array's name is only a host-side stand-in, never a device pointer.
gqa_status scratch_for_current_device(float **scratch, int *num_sms)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GQA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_na_mu);
    if (!g_scratch_addr[dev]) {
        float *p = nullptr;
        if (cudaGetSymbolAddress(reinterpret_cast<void **>(&p), g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return GQA_ERR_CUDA;
        }
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
            return GQA_ERR_CUDA;
        g_scratch_addr[dev] = p;
        g_num_sms[dev] = sms;
    }
    if (!g_na_encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return GQA_ERR_CUDA;
        g_na_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    *scratch = g_scratch_addr[dev];
    *num_sms = g_num_sms[dev];
    return GQA_OK;
}

// [B][Tmax][Hkv][d] bf16 cache, boxes of `rows` rows of one 64-column half, 128-byte swizzle.
gqa_status encode_cache_map(CUtensorMap *tm, const void *base, int B, int Tmax, int Hkv, int rows)
{
    const uint64_t d = kHeadDim;
    cuuint64_t dims[4] = {d, (cuuint64_t)Hkv, (cuuint64_t)Tmax, (cuuint64_t)B};
    cuuint64_t strides[3] = {d * 2, d * Hkv * 2, d * Hkv * (uint64_t)Tmax * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = g_na_encode(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box,
                             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? GQA_OK : GQA_ERR_CUDA;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" gqa_status gqa_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                         const int32_t *seqlens, int B, int Hq, int Hkv, int d, int Tmax, float scale,
                                         void *out, void *stream)
{
    set_last_launch_count(0);
    if (!q || !k_cache || !v_cache || !seqlens || !out) return GQA_ERR_INVALID_ARG;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || Tmax <= 0 || Hq % Hkv != 0) return GQA_ERR_INVALID_ARG;
    if (d != kHeadDim || B > 65535) return GQA_ERR_UNSUPPORTED;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
        !aligned(seqlens, 4))
        return GQA_ERR_MISALIGNED;

    float *scratch = nullptr;
    int num_sms = 0;
    gqa_status s = scratch_for_current_device(&scratch, &num_sms);
    if (s != GQA_OK) return s;

    int chunk = 0, nsplit = 0;
    size_t need = 0;
    if ((s = gqa_decode_plan(B, Hq, Hkv, d, Tmax, num_sms, &chunk, &nsplit, &need)) != GQA_OK) return s;
    if (need > kScratchBytes) return GQA_ERR_UNSUPPORTED;   // partials would not fit the fixed scratch
    const int g = Hq / Hkv;
    const DecodeShape sh = decode_shape(g);
    const int nhb = sh.nhb;
    if ((long long)Hkv * nhb > 65535) return GQA_ERR_UNSUPPORTED;

    CUtensorMap tmK, tmV;
    if ((s = encode_cache_map(&tmK, k_cache, B, Tmax, Hkv, sh.tile)) != GQA_OK) return s;
    if ((s = encode_cache_map(&tmV, v_cache, B, Tmax, Hkv, sh.tile)) != GQA_OK) return s;

    DecodeArgs a;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.seqlens = seqlens;
    a.out = static_cast<__nv_bfloat16 *>(out);
    // every split the combine reads is written by this call's split kernel first, so
    // nothing in the scratch has to start at zero
    a.part_o = scratch;
    a.part_ml = scratch + (size_t)B * Hq * nsplit * kHeadDim;
    a.status = device_status_word();
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.Tmax = Tmax;
    a.group = g;
    a.chunk = chunk;
    a.nsplit = nsplit;
    a.nhb = nhb;
    a.qscale = scale * 1.4426950408889634f;
    a.wait_budget_ns = 1000000000ull;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (launch_decode_split(tmK, tmV, a, st) != cudaSuccess) return GQA_ERR_CUDA;
    int n = 1;
    if (nsplit > 1) {
        if (launch_decode_combine(a, st) != cudaSuccess) return GQA_ERR_CUDA;
        ++n;
    }
    set_last_launch_count(n);
    return GQA_OK;
}
