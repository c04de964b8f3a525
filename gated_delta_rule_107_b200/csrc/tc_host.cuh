// tc_host.cuh -- host helpers of the tensor-core path: TMA tensor-map encoding.
//
// cuTensorMapEncodeTiled is a driver-API function; it is looked up at run time
// through cudaGetDriverEntryPoint so that the library does not link libcuda.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dr {
namespace tc {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)p;
    }
    return fn;
}

// Tensor map over a contiguous bf16 tensor [D3][D2][D1][D0] (D0 innermost), with a
// box of (64, 1, box_rows, 1) elements and 128-byte swizzle: one load brings 64
// consecutive innermost elements of `box_rows` consecutive D2 indices at fixed
// (D1, D3) -- e.g. 64 channels of 64 tokens of one head of one batch for a
// [B, T, H, d] tensor.  Out-of-range rows are zero-filled.
inline bool make_map_4d_bf16(CUtensorMap *map, const void *base, uint64_t D0, uint64_t D1, uint64_t D2, uint64_t D3,
                             uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {D0, D1, D2, D3};
    const cuuint64_t strides[3] = {D0 * 2, D0 * D1 * 2, D0 * D1 * D2 * 2};
    const cuuint32_t box[4] = {64, 1, box_rows, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Tensor map over a row-major bf16 matrix [D1][D0] (D0 innermost, a multiple of 8),
// with a box of 64 x box_rows elements and 128-byte swizzle.
inline bool make_map_2d_bf16(CUtensorMap *map, const void *base, uint64_t D0, uint64_t D1, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {D0, D1};
    const cuuint64_t strides[1] = {D0 * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace tc
}  // namespace dr
