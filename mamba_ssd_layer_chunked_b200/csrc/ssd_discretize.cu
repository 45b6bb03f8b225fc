// ssd_discretize.cu -- the step before the SSD scan in the Mamba block: the
// input-dependent step size and the discretisation of A and B x.
//
//   delta = softplus(dt + dt_bias[h]),   log a = delta * A[h]
//   X = s * x  with  s = delta                       (Euler for B: B_bar = delta B)
//                 or s = (exp(delta A) - 1) / A      (zero-order hold for B)
//
// Source: the Mamba page (ai.tomabc.com, paper story 21): delta = softplus(
// linear(x) + bias) in the block pseudocode and A_bar = exp(delta * A); "Mamba
// and state space models" (wang-x-xia.github.io), section 2: the zero-order-hold
// discretisation h_t = A_bar h_{t-1} + B_bar x_t. The per-head scalar s is put
// on x (B is shared by the heads of a group), which the recurrence does not
// distinguish from putting it on B. Bandwidth-bound: x in, X out.

#include "ssd_common.cuh"

namespace ssd {

namespace {

constexpr int kDiscThreads = 256;
constexpr int kDiscVec = 2;  // 16-byte vectors per thread

__device__ __forceinline__ float softplus_f(float z) { return z > 20.f ? z : log1pf(expf(z)); }

template <typename T>
struct Vec16;  // 16 bytes of T: 8 bf16 or 4 fp32
template <>
struct Vec16<__nv_bfloat16> {
    static constexpr int kN = 8;
};
template <>
struct Vec16<float> {
    static constexpr int kN = 4;
};

// each thread takes kDiscVec 16-byte vectors (8 bf16 or 4 fp32 elements of a
// row (b, t, h) of P elements), 256 vectors apart; a row's delta is recomputed
// by each thread that touches it (cheaper than sharing it: the kernel is bound
// by the bytes of x and X)
template <typename T, typename I>
__global__ void __launch_bounds__(kDiscThreads) discretize_kernel(int64_t rows, int nheads, int headdim,
                                                                  const float* __restrict__ dt,
                                                                  const float* __restrict__ dt_bias,
                                                                  const float* __restrict__ A, const T* __restrict__ x,
                                                                  int zoh, float* __restrict__ log_a, T* __restrict__ X) {
    constexpr int V = Vec16<T>::kN;
    // I: 32-bit index arithmetic where the element count allows (a 64-bit
    // division by a runtime divisor costs several times the rest of the thread)
    const I PV = (I)(headdim / V);
    const I n = (I)rows * PV;
    // kDiscVec vectors per thread, every load issued before any is used
    const I i0 = (I)blockIdx.x * (kDiscVec * kDiscThreads) + threadIdx.x;
    uint4 inv[kDiscVec];
#pragma unroll
    for (int u = 0; u < kDiscVec; ++u) {
        const I i = i0 + (I)u * kDiscThreads;
        if (i < n) inv[u] = __ldcs(reinterpret_cast<const uint4*>(x) + i);
    }
#pragma unroll
    for (int u = 0; u < kDiscVec; ++u) {
        const I i = i0 + (I)u * kDiscThreads;
        if (i >= n) break;
        const I r = i / PV;
        const int q = (int)(i - r * PV);
        const int h = (int)(r % (I)nheads);
        const float a = A[h];
        const float delta = softplus_f(dt[r] + (dt_bias ? dt_bias[h] : 0.f));
        const float la = delta * a;
        if (q == 0) log_a[r] = la;
        const float s = zoh ? (a != 0.f ? expm1f(la) / a : delta) : delta;
        const uint4 in = inv[u];
        uint4 out;
        if constexpr (V == 8) {
            const __nv_bfloat162* xi = reinterpret_cast<const __nv_bfloat162*>(&in);
            __nv_bfloat162* xo = reinterpret_cast<__nv_bfloat162*>(&out);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(xi[e]);
                xo[e] = __floats2bfloat162_rn(s * f.x, s * f.y);
            }
        } else {
            const float* xi = reinterpret_cast<const float*>(&in);
            float* xo = reinterpret_cast<float*>(&out);
#pragma unroll
            for (int e = 0; e < 4; ++e) xo[e] = s * xi[e];
        }
        __stcs(reinterpret_cast<uint4*>(X) + i, out);
    }
}

}  // namespace

cudaError_t launch_discretize(int64_t rows, int nheads, int headdim, ssd_dtype dt_x, const float* dt,
                              const float* dt_bias, const float* A, const void* x, int zoh, float* log_a, void* X,
                              cudaStream_t st) {
    const int64_t n = rows * (headdim / (dt_x == SSD_DTYPE_F32 ? 4 : 8));
    const unsigned grid = (unsigned)((n + kDiscVec * kDiscThreads - 1) / (kDiscVec * kDiscThreads));
    const bool i32 = n + kDiscVec * kDiscThreads <= (int64_t)UINT32_MAX;
    if (dt_x == SSD_DTYPE_F32) {
        auto k = i32 ? discretize_kernel<float, uint32_t> : discretize_kernel<float, int64_t>;
        k<<<grid, kDiscThreads, 0, st>>>(rows, nheads, headdim, dt, dt_bias, A, (const float*)x, zoh, log_a,
                                         (float*)X);
    } else {
        auto k = i32 ? discretize_kernel<__nv_bfloat16, uint32_t> : discretize_kernel<__nv_bfloat16, int64_t>;
        k<<<grid, kDiscThreads, 0, st>>>(rows, nheads, headdim, dt, dt_bias, A, (const __nv_bfloat16*)x, zoh,
                                         log_a, (__nv_bfloat16*)X);
    }
    return cudaGetLastError();
}

}  // namespace ssd
