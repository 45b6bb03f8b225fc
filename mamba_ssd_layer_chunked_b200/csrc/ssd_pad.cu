// ssd_pad.cu -- state-dimension slicing for the fused path of ssd_fwd.
//
// The rows n of the state evolve independently: H_t[n, :] = a_t H_{t-1}[n, :] +
// B_t[n] x_t^T, and y_t = sum_n C_t[n] H_t[n, :] + D x_t (the recurrence of
// "Mamba-2: writing the recurrent state as a structured matrix", wq-win section
// 2.1, read row by row). So a problem with dstate N is the sum over slices of n
// of problems on those slices (D counted once), and a slice padded with zero
// columns of B and C has zero extra state rows and unchanged outputs. These
// kernels copy a slice of B / C / states into a padded buffer and copy states
// back; the scan of a later slice adds its Y to the output in its epilogue.

#include "ssd_common.cuh"

namespace ssd {

namespace {

constexpr int kPadThreads = 256;

// dst[r, j] = j < w ? src[r, n0 + j] : 0, rows of N (src) and Np (dst) elements
template <typename T>
__global__ void pad_rows_kernel(const T* __restrict__ src, T* __restrict__ dst, int64_t rows, int N, int n0, int w,
                                int Np) {
    const int64_t i = (int64_t)blockIdx.x * kPadThreads + threadIdx.x;
    if (i >= rows * Np) return;
    const int64_t r = i / Np;
    const int j = (int)(i % Np);
    dst[i] = j < w ? src[r * N + n0 + j] : T(0.f);
}

// states: src [S, N, P] -> dst [S, Np, P] rows n0 .. n0+w-1 (zero rows after)
__global__ void pad_states_kernel(const float* __restrict__ src, float* __restrict__ dst, int64_t S, int N, int n0,
                                  int w, int Np, int P) {
    const int64_t i = (int64_t)blockIdx.x * kPadThreads + threadIdx.x;
    if (i >= S * Np * P) return;
    const int p = (int)(i % P);
    const int64_t rest = i / P;
    const int j = (int)(rest % Np);
    const int64_t s = rest / Np;
    dst[i] = j < w ? src[(s * N + n0 + j) * P + p] : 0.f;
}

// states back: dst [S, N, P] rows n0 .. n0+w-1 <- src [S, Np, P] rows 0 .. w-1
__global__ void unpad_states_kernel(const float* __restrict__ src, float* __restrict__ dst, int64_t S, int N, int n0,
                                    int w, int Np, int P) {
    const int64_t i = (int64_t)blockIdx.x * kPadThreads + threadIdx.x;
    if (i >= S * (int64_t)w * P) return;
    const int p = (int)(i % P);
    const int64_t rest = i / P;
    const int j = (int)(rest % w);
    const int64_t s = rest / w;
    dst[(s * N + n0 + j) * P + p] = src[(s * Np + j) * P + p];
}

unsigned blocks_for(int64_t n) { return (unsigned)((n + kPadThreads - 1) / kPadThreads); }

}  // namespace

cudaError_t launch_pad_bc(const void* src, void* dst, int64_t rows, int N, int n0, int w, int Np, cudaStream_t st) {
    pad_rows_kernel<__nv_bfloat16><<<blocks_for(rows * Np), kPadThreads, 0, st>>>(
        (const __nv_bfloat16*)src, (__nv_bfloat16*)dst, rows, N, n0, w, Np);
    return cudaGetLastError();
}

cudaError_t launch_pad_states(const float* src, float* dst, int64_t S, int N, int n0, int w, int Np, int P,
                              cudaStream_t st) {
    pad_states_kernel<<<blocks_for(S * Np * P), kPadThreads, 0, st>>>(src, dst, S, N, n0, w, Np, P);
    return cudaGetLastError();
}

cudaError_t launch_unpad_states(const float* src, float* dst, int64_t S, int N, int n0, int w, int Np, int P,
                                cudaStream_t st) {
    unpad_states_kernel<<<blocks_for(S * (int64_t)w * P), kPadThreads, 0, st>>>(src, dst, S, N, n0, w, Np, P);
    return cudaGetLastError();
}

}  // namespace ssd
