// ssd_tmap.cu -- TMA tensor maps of the tensor-core kernels: 4-D bf16 maps
// over the [batch, token, head or group, inner] tensors X, Y, B and C, with
// 128-byte swizzle, encoded through the driver entry point.

#include <cuda.h>

#include <mutex>

#include "ssd_tc.cuh"

namespace ssd {

// ---------------------------------------------------------------------------
// host: tensor maps
// ---------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

// 4-D bf16 map over a [batch][token][mid][inner] row-major tensor, addressed as
// (inner, mid, token, batch) = (d0, d1, d2, d3) so the strides increase; a box
// is 64 inner elements (128 bytes, 128-byte swizzle) x 1 x box_tok tokens x 1.
cudaError_t make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t tokens,
                     uint64_t batch, uint32_t box_tok) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[4] = {inner, mid, tokens, batch};
    const cuuint64_t strides[3] = {inner * 2, mid * inner * 2, tokens * mid * inner * 2};
    const cuuint32_t box[4] = {64, 1, box_tok, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t x_map(CUtensorMap* m, const Dims& d, const void* X, uint32_t box_tok) {
    return make_map(m, X, d.headdim, d.nheads, d.seqlen, d.batch, box_tok);
}

cudaError_t bc_map(CUtensorMap* m, const Dims& d, const void* Bp, uint32_t box_tok) {
    return make_map(m, Bp, d.dstate, d.ngroups, d.seqlen, d.batch, box_tok);
}

}  // namespace ssd
