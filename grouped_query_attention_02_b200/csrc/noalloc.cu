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
#include <mutex>

#include "../../include/gqa.h"
#include "internal.h"

namespace {

using namespace gqa;

constexpr size_t kScratchBytes = size_t(32) << 20;   // 32 MiB of split partials per device
static __device__ __align__(256) float g_noalloc_scratch[kScratchBytes / sizeof(float)];

constexpr int kMaxDevices = 64;
std::mutex g_na_mu;
uint8_t *g_scratch_addr[kMaxDevices] = {};           // device address of the array, per device
int g_num_sms[kMaxDevices] = {};

// Once per device, with that device current: the array's device address.  In host
// code the array's name is only a host-side stand-in, never a device pointer.
gqa_status scratch_for_current_device(uint8_t **scratch, int *num_sms)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GQA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_na_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return GQA_ERR_CUDA;
        }
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
            return GQA_ERR_CUDA;
        g_scratch_addr[dev] = static_cast<uint8_t *>(p);
        g_num_sms[dev] = sms;
    }
    *scratch = g_scratch_addr[dev];
    *num_sms = g_num_sms[dev];
    return GQA_OK;
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

    uint8_t *scratch = nullptr;
    int num_sms = 0;
    gqa_status s = scratch_for_current_device(&scratch, &num_sms);
    if (s != GQA_OK) return s;
    // the same plan as gqa_decode; its workspace must fit the fixed array.  Every piece of
    // scratch the kernels read is written earlier in the same call (the plan, then the
    // partials), so nothing in it has to start at zero.
    const DecodePlan p = decode_plan_host(B, Hq, Hkv, Tmax, num_sms, kScratchBytes - (size_t(1) << 20));
    if (p.ws_bytes > kScratchBytes) return GQA_ERR_UNSUPPORTED;
    int *status = device_status_word();
    if (!status) return GQA_ERR_CUDA;
    int launches = 0;
    s = static_cast<gqa_status>(decode_enqueue(q, k_cache, v_cache, seqlens, B, Hq, Hkv, Tmax, scale, out,
                                               p.ws_bytes ? scratch : nullptr, p, num_sms, status,
                                               static_cast<cudaStream_t>(stream), &launches, nullptr, nullptr));
    set_last_launch_count(launches);
    return s;
}
