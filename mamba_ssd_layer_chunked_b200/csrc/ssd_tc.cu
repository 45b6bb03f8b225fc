// ssd_tc.cu -- tcgen05 kernels (placeholder until the tensor-core kernels land:
// every problem routes to the SIMT kernels).
#include "ssd_tc.cuh"

namespace ssd {

bool tc_supported(const ssd_problem*) { return false; }

cudaError_t launch_chunk_state_tc(const Dims&, const void*, const void*, const float*, const int32_t*, float*,
                                  float*, cudaStream_t) {
    return cudaErrorNotSupported;
}

cudaError_t launch_chunk_scan_tc(const Dims&, const void*, const void*, const void*, const float*, const float*,
                                 const float*, const float*, const int32_t*, void*, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace ssd
