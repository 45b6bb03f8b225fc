// ssd_common.cuh -- internal helpers shared by the CUDA translation units of
// libssd_b200.so. Not part of the C ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ssd.h"

namespace ssd {

// Problem sizes as the kernels see them (validated on the host first).
struct Dims {
    int batch, seqlen, nheads, headdim, dstate, ngroups, chunk, nseq, nchunks;
    int heads_per_group;
};

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// Sequence id of token t of batch row b, clamped to [0, nseq) so that
// out-of-contract ids can never index outside init/final state buffers.
__device__ __forceinline__ int seq_at(const int32_t* seq_idx, int64_t row_off, int t, int nseq) {
    if (!seq_idx) return 0;
    int s = seq_idx[row_off + t];
    return s < 0 ? 0 : (s >= nseq ? nseq - 1 : s);
}

// the id of token t of a chunk position that may lie past the row end: the
// positions after the last token of a partial last chunk take the last token's
// id, so that they extend its sequence piece (with log a = 0 and x = B = C = 0
// they change no state and no output)
__device__ __forceinline__ int seq_at_padded(const int32_t* seq_idx, int64_t row_off, int t, int seqlen, int nseq) {
    return seq_at(seq_idx, row_off, t < seqlen ? t : seqlen - 1, nseq);
}

// Flat offsets (int64 so that large problems cannot overflow).
__host__ __device__ __forceinline__ int64_t x_off(const Dims& d, int b, int t, int h) {
    return (((int64_t)b * d.seqlen + t) * d.nheads + h) * d.headdim;
}
__host__ __device__ __forceinline__ int64_t bc_off(const Dims& d, int b, int t, int g) {
    return (((int64_t)b * d.seqlen + t) * d.ngroups + g) * d.dstate;
}
__host__ __device__ __forceinline__ int64_t cs_off(const Dims& d, int b, int h, int c) {
    return (((int64_t)b * d.nheads + h) * d.nchunks + c) * d.chunk;
}
// state buffers [batch, nchunks, nheads, dstate, headdim]
__host__ __device__ __forceinline__ int64_t st_off(const Dims& d, int b, int c, int h) {
    return (((int64_t)b * d.nchunks + c) * d.nheads + h) * (int64_t)d.dstate * d.headdim;
}
// per-sequence states [batch, nseq, nheads, dstate, headdim]
__host__ __device__ __forceinline__ int64_t seqst_off(const Dims& d, int b, int s, int h) {
    return (((int64_t)b * d.nseq + s) * d.nheads + h) * (int64_t)d.dstate * d.headdim;
}

// ---- launchers (host) ------------------------------------------------------

cudaError_t launch_discretize(int64_t rows, int nheads, int headdim, ssd_dtype dt_x, const float* dt,
                              const float* dt_bias, const float* A, const void* x, int zoh, float* log_a, void* X,
                              cudaStream_t st);

cudaError_t launch_decode_step(int batch, int nheads, int headdim, int dstate, int ngroups, ssd_dtype dt,
                               const void* x, const float* log_a, const void* B, const void* C, const float* D,
                               float* state, void* y, cudaStream_t st);

// The chunked steps take the within-chunk cumsum as fp32 (the step entry
// points) or fp64 (ssd_fwd's SIMT family, where exp(cs_k - cs_l) needs the
// difference to fp32 accuracy); the sums are formed in fp64 either way.
cudaError_t launch_chunk_cumsum(const Dims& d, const float* log_a, float* cs, cudaStream_t st);
cudaError_t launch_chunk_cumsum(const Dims& d, const float* log_a, double* cs, cudaStream_t st);

cudaError_t launch_chunk_state_simt(const Dims& d, ssd_dtype dt, const void* X, const void* B,
                                    const float* cs, const int32_t* seq_idx, float* states,
                                    float* final_states, cudaStream_t st);
cudaError_t launch_chunk_state_simt(const Dims& d, ssd_dtype dt, const void* X, const void* B,
                                    const double* cs, const int32_t* seq_idx, float* states,
                                    float* final_states, cudaStream_t st);

cudaError_t launch_state_passing(const Dims& d, const float* cs, const float* chunk_states,
                                 float* incoming, const float* init_states,
                                 const int32_t* seq_idx, float* final_states, cudaStream_t st);
cudaError_t launch_state_passing(const Dims& d, const double* cs, const float* chunk_states,
                                 float* incoming, const float* init_states,
                                 const int32_t* seq_idx, float* final_states, cudaStream_t st);

cudaError_t launch_chunk_scan_simt(const Dims& d, ssd_dtype dt, const void* X, const void* B,
                                   const void* C, const float* cs, const float* D,
                                   const float* incoming, const float* init_states,
                                   const int32_t* seq_idx, void* Y, cudaStream_t st);
cudaError_t launch_chunk_scan_simt(const Dims& d, ssd_dtype dt, const void* X, const void* B,
                                   const void* C, const double* cs, const float* D,
                                   const float* incoming, const float* init_states,
                                   const int32_t* seq_idx, void* Y, cudaStream_t st);

// Sets cudaFuncAttributeMaxDynamicSharedMemorySize once per (kernel, device).
cudaError_t ensure_smem_attr(const void* func, int bytes, int slot);

// Device address of the library's error word on the current device (looked up
// once per device): kernels with bounded waits OR a code into it when a wait
// gives up; ssd_device_error reads and clears it.
cudaError_t device_error_word(unsigned int** out);

}  // namespace ssd
