// tma_encode.cuh -- the driver's cuTensorMapEncodeTiled, looked up once through
// the runtime (no link-time dependency on libcuda), shared by the entry points
// that build TMA descriptors.  Internal.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <mutex>

namespace dsa {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn tma_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// A bf16 operand of the dense GEMM as a 3-D map: element (k, r, b) at base +
// b * batch_stride + r * row_stride + k (strides in elements, multiples of 8),
// 128-byte swizzle, reads past K or rows fill with zeros.  The two outer
// dimensions are ordered by stride: {K, rows, batch} with boxes {64, box_rows,
// 1}, or, when the batch stride is the smaller one (heads interleaved inside a
// row of tokens), {K, batch, rows} with boxes {64, 1, box_rows} -- the same
// shared-memory tile either way.  *batch_inner tells which.
inline bool encode_gemm_operand(CUtensorMap *map, const void *base, int64_t K, int64_t rows, int64_t batch,
                                int64_t row_stride, int64_t batch_stride, int box_rows, int *batch_inner) {
    EncodeTiledFn enc = tma_encode_fn();
    if (!enc) return false;
    const bool inner = batch > 1 && batch_stride < row_stride;
    *batch_inner = inner ? 1 : 0;
    const int64_t bstride = batch > 1 ? batch_stride : row_stride * rows;
    cuuint64_t dims[3], strides[2];
    cuuint32_t box[3];
    dims[0] = static_cast<cuuint64_t>(K);
    box[0] = 64;
    if (inner) {
        dims[1] = static_cast<cuuint64_t>(batch);
        dims[2] = static_cast<cuuint64_t>(rows);
        strides[0] = static_cast<cuuint64_t>(bstride * 2);
        strides[1] = static_cast<cuuint64_t>(row_stride * 2);
        box[1] = 1;
        box[2] = static_cast<cuuint32_t>(box_rows);
    } else {
        dims[1] = static_cast<cuuint64_t>(rows);
        dims[2] = static_cast<cuuint64_t>(batch);
        strides[0] = static_cast<cuuint64_t>(row_stride * 2);
        strides[1] = static_cast<cuuint64_t>(bstride * 2);
        box[1] = static_cast<cuuint32_t>(box_rows);
        box[2] = 1;
    }
    cuuint32_t es[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace dsa
