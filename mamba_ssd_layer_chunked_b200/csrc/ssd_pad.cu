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

// One thread per 16 bytes (8 bf16 of B / C, 4 fp32 of a state row); N, n0, w
// and Np are multiples of 16 and P of 4, so every vector lies inside or
// outside the slice as a whole. I is the index type: 32-bit where the vector
// count fits (a 64-bit division by a runtime divisor costs several times the
// rest of the thread).

// dst[r, j] = j < w ? src[r, n0 + j] : 0, rows of N (src) and Np (dst) bf16
template <typename I>
__global__ void pad_rows_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, I nvec, int N, int n0, int w,
                                int Np) {
    const I i = (I)blockIdx.x * kPadThreads + threadIdx.x;
    if (i >= nvec) return;
    const I np8 = (I)(Np / 8);
    const I r = i / np8;
    const int j = 8 * (int)(i - r * np8);
    dst[i] = j < w ? src[(r * (I)N + (I)(n0 + j)) / 8] : make_uint4(0u, 0u, 0u, 0u);
}

// states: src [S, N, P] -> dst [S, Np, P] rows n0 .. n0+w-1 (zero rows after)
template <typename I>
__global__ void pad_states_kernel(const float4* __restrict__ src, float4* __restrict__ dst, I nvec, int N, int n0,
                                  int w, int Np, int P) {
    const I i = (I)blockIdx.x * kPadThreads + threadIdx.x;
    if (i >= nvec) return;
    const I p4 = (I)(P / 4);
    const I rest = i / p4;
    const I q = i - rest * p4;
    const I s = rest / (I)Np;
    const int j = (int)(rest - s * (I)Np);
    dst[i] = j < w ? src[(s * (I)N + (I)(n0 + j)) * p4 + q] : make_float4(0.f, 0.f, 0.f, 0.f);
}

// states back: dst [S, N, P] rows n0 .. n0+w-1 <- src [S, Np, P] rows 0 .. w-1
template <typename I>
__global__ void unpad_states_kernel(const float4* __restrict__ src, float4* __restrict__ dst, I nvec, int N, int n0,
                                    int w, int Np, int P) {
    const I i = (I)blockIdx.x * kPadThreads + threadIdx.x;
    if (i >= nvec) return;
    const I p4 = (I)(P / 4);
    const I rest = i / p4;
    const I q = i - rest * p4;
    const I s = rest / (I)w;
    const int j = (int)(rest - s * (I)w);
    dst[(s * (I)N + (I)(n0 + j)) * p4 + q] = src[(s * (I)Np + (I)j) * p4 + q];
}

unsigned blocks_for(int64_t n) { return (unsigned)((n + kPadThreads - 1) / kPadThreads); }

// 32-bit indices when every index the kernel forms (vectors and source offsets
// of either side, in elements) stays below 2^32
bool fits32(int64_t a, int64_t b) { return a + kPadThreads < (int64_t)UINT32_MAX && b < (int64_t)UINT32_MAX; }

}  // namespace

cudaError_t launch_pad_bc(const void* src, void* dst, int64_t rows, int N, int n0, int w, int Np, cudaStream_t st) {
    const int64_t nvec = rows * Np / 8;
    if (nvec == 0) return cudaSuccess;
    const auto s = (const uint4*)src;
    const auto d = (uint4*)dst;
    if (fits32(nvec, rows * N))
        pad_rows_kernel<uint32_t><<<blocks_for(nvec), kPadThreads, 0, st>>>(s, d, (uint32_t)nvec, N, n0, w, Np);
    else
        pad_rows_kernel<int64_t><<<blocks_for(nvec), kPadThreads, 0, st>>>(s, d, nvec, N, n0, w, Np);
    return cudaGetLastError();
}

cudaError_t launch_pad_states(const float* src, float* dst, int64_t S, int N, int n0, int w, int Np, int P,
                              cudaStream_t st) {
    const int64_t nvec = S * Np * P / 4;
    if (nvec == 0) return cudaSuccess;
    const auto s = (const float4*)src;
    const auto d = (float4*)dst;
    if (fits32(nvec, S * N * P))
        pad_states_kernel<uint32_t><<<blocks_for(nvec), kPadThreads, 0, st>>>(s, d, (uint32_t)nvec, N, n0, w, Np, P);
    else
        pad_states_kernel<int64_t><<<blocks_for(nvec), kPadThreads, 0, st>>>(s, d, nvec, N, n0, w, Np, P);
    return cudaGetLastError();
}

cudaError_t launch_unpad_states(const float* src, float* dst, int64_t S, int N, int n0, int w, int Np, int P,
                                cudaStream_t st) {
    const int64_t nvec = S * (int64_t)w * P / 4;
    if (nvec == 0) return cudaSuccess;
    const auto s = (const float4*)src;
    const auto d = (float4*)dst;
    if (fits32(nvec, S * (N > Np ? N : Np) * P))
        unpad_states_kernel<uint32_t><<<blocks_for(nvec), kPadThreads, 0, st>>>(s, d, (uint32_t)nvec, N, n0, w, Np,
                                                                                P);
    else
        unpad_states_kernel<int64_t><<<blocks_for(nvec), kPadThreads, 0, st>>>(s, d, nvec, N, n0, w, Np, P);
    return cudaGetLastError();
}

}  // namespace ssd
