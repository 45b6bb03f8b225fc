// ssd_waitcheck.cu -- a self-test of the bounded waits' failure report.
//
// The tensor-core kernels wait on shared-memory barriers; each wait gives up
// after a time limit and lets its CTA run to its end, which then sets a bit in
// the library's device error word (tc_ptx.cuh). This kernel makes that happen on
// purpose, with a short limit, on a barrier that nothing ever completes, so
// that a test can check the report reaches the host (ssd_device_error) and is
// cleared, and that the device stays usable. It issues no copies and no
// matrix products, so nothing is in flight when it gives up.

#include "ssd_common.cuh"
#include "tc_ptx.cuh"

namespace {

using namespace ssd::tc;

__global__ void __launch_bounds__(32) wait_timeout_kernel(uint64_t limit_ns, unsigned int* err) {
    __shared__ __align__(8) uint64_t bar;
    wait_guard_init(err);
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // one arrival completes phase 0; none ever comes
        mbar_fence_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // gives up after limit_ns and reports; the second wait then returns at
        // once (the CTA is marked), as later waits of a failed kernel do
        if (!mbar_wait(&bar, 0, limit_ns)) mbar_wait(&bar, 0, limit_ns);
    }
    __syncthreads();
    wait_guard_finish();
}

}  // namespace

extern "C" ssd_status ssd_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
    if (limit_ns < 1000ull || limit_ns > 1000000000ull) return SSD_ERR_INVALID_ARG;  // 1 us .. 1 s
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
        cudaGetLastError();
        return SSD_ERR_UNSUPPORTED;
    }
    if (major != 10) return SSD_ERR_UNSUPPORTED;
    unsigned int* err = nullptr;
    if (ssd::device_error_word(&err) != cudaSuccess) {
        cudaGetLastError();
        return SSD_ERR_CUDA;
    }
    wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(limit_ns, err);
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
