// ssd_noalloc.cu -- ssd_fwd_noalloc: the forward pass for callers that cannot
// allocate device memory.
//
// Some callers may not call cudaMalloc at all: hosts that plan every byte of
// device memory up front (inference servers, plugin hosts that own the
// allocator) and latency-critical loops where an allocation's implicit device
// synchronisation is not acceptable. They still own inputs and outputs, but
// cannot provide ssd_fwd's workspace. This entry point takes its scratch from a
// fixed array in the library's own device memory instead, so it allocates
// nothing per call.
//
// The array below is reserved on every GPU where this module is loaded (at the
// latest on the first call of the entry point on that GPU) and stays reserved
// until the process exits. Its device address is looked up once per device
// (cudaGetSymbolAddress with that device current); make that first call before
// any stream capture. All calls share the array: calls whose kernels overlap on
// the GPU (different streams, or other threads) race on it and must be ordered
// by the caller. The array keeps whatever the last call left in it; the pipeline
// writes every scratch byte it reads, so nothing has to start at zero.

#include <cuda_runtime.h>

#include <mutex>

#include "ssd.h"

static __device__ __align__(256) unsigned char g_ssd_noalloc_scratch[SSD_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
ssd_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return SSD_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return SSD_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_ssd_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return SSD_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return SSD_OK;
}

}  // namespace

extern "C" ssd_status ssd_fwd_noalloc(const ssd_problem* p, const void* X, const float* log_a, const void* B,
                                      const void* C, const float* D, const float* init_states,
                                      const int32_t* seq_idx, void* Y, float* final_states, void* stream) {
    const size_t need = ssd_fwd_workspace_bytes(p);
    if (need == (size_t)-1) {
        const ssd_status s = ssd_check_problem(p);
        return s == SSD_OK ? SSD_ERR_INVALID_ARG : s;
    }
    if (need > SSD_NOALLOC_SCRATCH_BYTES) return SSD_ERR_WORKSPACE;  // larger than the fixed scratch
    const ssd_status s = ssd_check_problem(p);
    if (s != SSD_OK) return s;
    void* scratch = nullptr;
    const ssd_status a = scratch_address(&scratch);
    if (a != SSD_OK) return a;
    return ssd_fwd(p, X, log_a, B, C, D, init_states, seq_idx, Y, final_states, scratch,
                   SSD_NOALLOC_SCRATCH_BYTES, stream);
}
