// ssd_tc.cuh -- tensor-core (tcgen05 / TMEM / TMA) kernels of the SSD chunked
// scan for sm_100a: chunk_state and chunk_scan. Internal, not part of the C ABI.
#pragma once

#include <cuda.h>

#include "ssd_common.cuh"

namespace ssd {

// TMA tensor maps (bf16, 128-byte swizzle, boxes of 64 x 1 x box_tok x 1)
cudaError_t x_map(CUtensorMap* m, const Dims& d, const void* X, uint32_t box_tok);
cudaError_t bc_map(CUtensorMap* m, const Dims& d, const void* Bp, uint32_t box_tok);

// True when the tcgen05 kernels cover problem p (dtype, head/state sizes, chunk).
bool tc_supported(const ssd_problem* p);

cudaError_t launch_chunk_state_tc(const Dims& d, const void* X, const void* B, const float* cs,
                                  const int32_t* seq_idx, float* states, float* final_states,
                                  cudaStream_t st);

cudaError_t launch_chunk_scan_tc(const Dims& d, const void* X, const void* B, const void* C,
                                 const float* cs, const float* D, const float* incoming,
                                 const float* init_states, const int32_t* seq_idx, void* Y,
                                 cudaStream_t st);

// ---- fused path (ssd_fused.cu) ----
bool fused_supported(const ssd_problem* p);
// segment length chosen for problem d on the current device (multiple of 128)
int fused_default_seglen(const Dims& d);
bool fused_seglen_ok(const Dims& d, int64_t seglen);
size_t fused_workspace_bytes(const Dims& d, int seglen);

cudaError_t launch_segment_state(const Dims& d, int seglen, const void* X, const float* log_a, const void* B,
                                 const int32_t* seq_idx, float* seg_states, float* seg_decay, cudaStream_t st);
cudaError_t launch_segment_passing(const Dims& d, int seglen, float* seg_states, const float* seg_decay,
                                   const float* init_states, const int32_t* seq_idx, cudaStream_t st);
cudaError_t launch_fused_scan(const Dims& d, int seglen, const void* X, const float* log_a, const void* B,
                              const void* C, const float* D, const float* seg_incoming, const float* init_states,
                              const int32_t* seq_idx, void* Y, float* final_states, cudaStream_t st);

}  // namespace ssd
