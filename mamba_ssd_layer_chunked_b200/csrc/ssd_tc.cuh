// ssd_tc.cuh -- the tensor-core (tcgen05 / TMEM / TMA) kernels of the SSD
// forward for sm_100a: the fused path's launchers and the TMA tensor maps they
// use. Internal, not part of the C ABI.
#pragma once

#include <cuda.h>

#include "ssd_common.cuh"

namespace ssd {

// TMA tensor maps (ssd_tmap.cu; bf16, 128-byte swizzle, boxes of 64 x 1 x box_tok x 1)
cudaError_t x_map(CUtensorMap* m, const Dims& d, const void* X, uint32_t box_tok);
cudaError_t bc_map(CUtensorMap* m, const Dims& d, const void* Bp, uint32_t box_tok);

// ---- fused path (ssd_fused.cu) ----
// The rows (batch row, head pair) x 128-token tiles laid end to end, cut into
// ranges of work_tiles tiles, one CTA each.
bool fused_supported(const ssd_problem* p);  // the step entry points: dstate 64 or 128
// ssd_fwd on the fused family: any dstate that is a multiple of 16 up to 256,
// as slices of at most 128 state rows padded to 64 or 128 (ssd_pad.cu)
bool fused_fwd_supported(const ssd_problem* p);
// tiles per range chosen for problem d on the current device
int fused_default_work_tiles(const Dims& d);
bool fused_work_ok(const Dims& d, int64_t work_tiles);
int64_t fused_work_count(const Dims& d, int64_t work_tiles);
// true when some range starts inside a row (then the cut states are needed)
bool fused_needs_cut_states(const Dims& d, int64_t work_tiles);
size_t fused_workspace_bytes(const Dims& d, int64_t work_tiles);

// row_ids non-null: one range per row (work_tiles = tiles per row), every
// row's state over its last sequence piece, and its first and last ids
cudaError_t launch_segment_state(const Dims& d, int64_t work_tiles, const void* X, const float* log_a, const void* B,
                                 const int32_t* seq_idx, float* work_local, float* work_decay, cudaStream_t st,
                                 int32_t* row_ids = nullptr);

// sequence parallelism (ssd_sp.cu)
cudaError_t launch_sp_combine(const Dims& d, int nranks, int rank, const float* g_loc, const float* g_dec,
                              const int32_t* g_ids, const float* init_states, float* init_local, cudaStream_t st);
cudaError_t launch_sp_own_finals(const Dims& d, int nranks, int rank, const int32_t* g_ids, float* final_states,
                                 cudaStream_t st);
// loc, dec, ids of a segment from the final states of its sequences from zero
// initial states (the chunked steps' output)
cudaError_t launch_sp_finish(const Dims& d, const float* log_a, const int32_t* seq_idx, const float* finals,
                             float* loc, float* dec, int32_t* ids, cudaStream_t st);
cudaError_t launch_segment_passing(const Dims& d, int64_t work_tiles, const float* work_local, const float* work_decay,
                                   const float* init_states, const int32_t* seq_idx, float* work_in, cudaStream_t st);
// work_in (the output of segment_passing) or, when it is null, work_local and
// work_decay (the output of segment_state): the kernel then chains the pieces
// before each range's cut itself
cudaError_t launch_fused_scan(const Dims& d, int64_t work_tiles, const void* X, const float* log_a, const void* B,
                              const void* C, const float* D, const float* work_in, const float* init_states,
                              const int32_t* seq_idx, void* Y, float* final_states, cudaStream_t st,
                              const float* work_local = nullptr, const float* work_decay = nullptr,
                              bool after_segment_state = false, const void* Yacc = nullptr);

// state-dimension slices (ssd_pad.cu)
cudaError_t launch_pad_bc(const void* src, void* dst, int64_t rows, int N, int n0, int w, int Np, cudaStream_t st);
cudaError_t launch_pad_states(const float* src, float* dst, int64_t S, int N, int n0, int w, int Np, int P,
                              cudaStream_t st);
cudaError_t launch_unpad_states(const float* src, float* dst, int64_t S, int N, int n0, int w, int Np, int P,
                                cudaStream_t st);

}  // namespace ssd
