// tcgen05 projection: placeholder until the tensor-core kernel lands.
#include "common.cuh"

namespace engram {

bool project_tc_supported(int64_t, int32_t, int32_t) { return false; }

cudaError_t launch_project_tc(const void*, int64_t, int32_t, const void*, const void*, const void*, const float*,
                              const float*, int32_t, void*, float*, uint32_t*, int, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace engram
