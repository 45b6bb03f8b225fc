// ssd_tc.cuh -- tensor-core (tcgen05 / TMEM / TMA) kernels of the SSD chunked
// scan for sm_100a: chunk_state and chunk_scan. Internal, not part of the C ABI.
#pragma once

#include "ssd_common.cuh"

namespace ssd {

// True when the tcgen05 kernels cover problem p (dtype, head/state sizes, chunk).
bool tc_supported(const ssd_problem* p);

cudaError_t launch_chunk_state_tc(const Dims& d, const void* X, const void* B, const float* cs,
                                  const int32_t* seq_idx, float* states, float* final_states,
                                  cudaStream_t st);

cudaError_t launch_chunk_scan_tc(const Dims& d, const void* X, const void* B, const void* C,
                                 const float* cs, const float* D, const float* incoming,
                                 const float* init_states, const int32_t* seq_idx, void* Y,
                                 cudaStream_t st);

}  // namespace ssd
