// prefill.cu -- causal GQA prefill on tcgen05 tensor cores (placeholder until the kernel lands).
#include "internal.h"
#include "ptx.cuh"

namespace gqa {

cudaError_t launch_prefill(const CUtensorMap &, const CUtensorMap &, const CUtensorMap &, const PrefillArgs &,
                           cudaStream_t)
{
    return cudaErrorNotSupported;
}

}  // namespace gqa
