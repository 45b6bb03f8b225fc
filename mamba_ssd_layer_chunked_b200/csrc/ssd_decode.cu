// ssd_decode.cu -- one step of the SSD recurrence per (batch row, head) with
// the state cached in fp32: the recurrent form used for token-by-token decoding.
//
//   H <- a H + B x^T,   y = C^T H + D x,   a = exp(log a)
//
// Source: "Mamba and state space models" (wang-x-xia.github.io, learn-ai/
// foundations), section 2 (the discrete recurrence with the D x skip term), and
// "Mamba-2: writing the recurrent state as a structured matrix"
// (wq-win.github.io/llm/088-mamba2.html), section 2.1 (the recurrence whose
// unrolled form the chunked scan computes). The step is bandwidth-bound: each
// head reads and writes its N x P fp32 state once; x, B, C, y are small.
//
// One CTA per (batch row, head). Thread (r, q) owns the 4 consecutive columns
// p = 4q .. 4q+3 of state rows n = r, r + R, r + 2R, ... (R row groups), so a
// warp reads and writes contiguous float4s; the read-out C^T H is reduced over
// the row groups in shared memory. A thread's rows are loaded together before
// they are updated (more bytes in flight), with streaming cache hints: each
// state row is read and written once per step.

#include "ssd_common.cuh"

namespace ssd {

namespace {

constexpr int kDecThreads = 128;  // small CTAs: 16 per SM, a finer last wave

template <typename T>
__device__ __forceinline__ float4 load4(const T* p);
template <>
__device__ __forceinline__ float4 load4<float>(const float* p) {
    return *reinterpret_cast<const float4*>(p);
}
template <>
__device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16* p) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    return make_float4(a.x, a.y, b.x, b.y);
}

template <typename T>
__device__ __forceinline__ void store4(T* p, float4 v);
template <>
__device__ __forceinline__ void store4<float>(float* p, float4 v) {
    *reinterpret_cast<float4*>(p) = v;
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* p, float4 v) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<const uint32_t*>(&a);
    u.y = *reinterpret_cast<const uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = u;
}

template <typename T>
__global__ void __launch_bounds__(kDecThreads) decode_step_kernel(int nheads, int headdim, int dstate, int heads_per_group,
                                                                  const T* __restrict__ x, const float* __restrict__ log_a,
                                                                  const T* __restrict__ B, const T* __restrict__ C,
                                                                  const float* __restrict__ D, float* __restrict__ state,
                                                                  T* __restrict__ y) {
    extern __shared__ float4 red[];  // [row groups][P / 4]
    const int bh = blockIdx.x;
    const int b = bh / nheads, h = bh % nheads;
    const int ngroups = nheads / heads_per_group, g = h / heads_per_group;
    const int P4 = headdim / 4, R = kDecThreads / P4;
    const int q = threadIdx.x % P4, r = threadIdx.x / P4;
    const float a = expf(log_a[bh]);
    const float4 xv = load4(x + (int64_t)bh * headdim + 4 * q);
    const T* Bb = B + ((int64_t)b * ngroups + g) * dstate;
    const T* Cb = C + ((int64_t)b * ngroups + g) * dstate;
    float* H = state + (int64_t)bh * dstate * headdim + 4 * q;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < R) {
        constexpr int kBatch = 8;  // state rows of this thread in flight at once
        for (int n0 = r; n0 < dstate; n0 += kBatch * R) {
            float4 hv[kBatch];
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                const int n = n0 + j * R;
                if (n < dstate) hv[j] = __ldcs(reinterpret_cast<const float4*>(H + (int64_t)n * headdim));
            }
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                const int n = n0 + j * R;
                if (n < dstate) {
                    const float bn = to_f32(Bb[n]), cn = to_f32(Cb[n]);
                    float4 h = hv[j];
                    h.x = fmaf(a, h.x, bn * xv.x);
                    h.y = fmaf(a, h.y, bn * xv.y);
                    h.z = fmaf(a, h.z, bn * xv.z);
                    h.w = fmaf(a, h.w, bn * xv.w);
                    __stcs(reinterpret_cast<float4*>(H + (int64_t)n * headdim), h);
                    acc.x = fmaf(cn, h.x, acc.x);
                    acc.y = fmaf(cn, h.y, acc.y);
                    acc.z = fmaf(cn, h.z, acc.z);
                    acc.w = fmaf(cn, h.w, acc.w);
                }
            }
        }
        red[r * P4 + q] = acc;
    }
    __syncthreads();
    if (r == 0) {
        float4 s = red[q];
        for (int j = 1; j < R; ++j) {
            const float4 t = red[j * P4 + q];
            s.x += t.x;
            s.y += t.y;
            s.z += t.z;
            s.w += t.w;
        }
        const float dh = D ? D[h] : 0.f;
        s.x = fmaf(dh, xv.x, s.x);
        s.y = fmaf(dh, xv.y, s.y);
        s.z = fmaf(dh, xv.z, s.z);
        s.w = fmaf(dh, xv.w, s.w);
        store4(y + (int64_t)bh * headdim + 4 * q, s);
    }
}

}  // namespace

cudaError_t launch_decode_step(int batch, int nheads, int headdim, int dstate, int ngroups, ssd_dtype dt,
                               const void* x, const float* log_a, const void* B, const void* C, const float* D,
                               float* state, void* y, cudaStream_t st) {
    const int P4 = headdim / 4, R = kDecThreads / P4;
    const size_t smem = (size_t)R * P4 * sizeof(float4);
    const dim3 grid(batch * nheads);
    const int hpg = nheads / ngroups;
    if (dt == SSD_DTYPE_F32)
        decode_step_kernel<float><<<grid, kDecThreads, smem, st>>>(
            nheads, headdim, dstate, hpg, (const float*)x, log_a, (const float*)B, (const float*)C, D, state, (float*)y);
    else
        decode_step_kernel<__nv_bfloat16><<<grid, kDecThreads, smem, st>>>(
            nheads, headdim, dstate, hpg, (const __nv_bfloat16*)x, log_a, (const __nv_bfloat16*)B,
            (const __nv_bfloat16*)C, D, state, (__nv_bfloat16*)y);
    return cudaGetLastError();
}

}  // namespace ssd
