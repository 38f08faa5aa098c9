// tma_encode.cuh -- the driver's cuTensorMapEncodeTiled, looked up once through
// the runtime (no link-time dependency on libcuda), shared by the entry points
// that build TMA descriptors.  Internal.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <cstring>
#include <mutex>

namespace dsa {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn tma_driver_encode_fn() {
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

// A tensor map is a pure function of its arguments, so the maps that every call
// re-encodes (the same caches, queries and shapes step after step) come from a
// small direct-mapped cache keyed on all of them; a miss encodes and fills the slot.
struct TmaEncodeKey {
    uint64_t base;
    uint64_t dims[5], strides[4];
    uint32_t box[5], es[5];
    uint32_t dtype, rank, interleave, swizzle, l2, oob;
};

inline CUresult tma_encode_cached(CUtensorMap *map, CUtensorMapDataType dtype, cuuint32_t rank, void *base,
                                  const cuuint64_t *dims, const cuuint64_t *strides, const cuuint32_t *box,
                                  const cuuint32_t *es, CUtensorMapInterleave il, CUtensorMapSwizzle sw,
                                  CUtensorMapL2promotion l2, CUtensorMapFloatOOBfill oob) {
    EncodeTiledFn real = tma_driver_encode_fn();
    if (!real) return CUDA_ERROR_NOT_INITIALIZED;
    if (rank < 1 || rank > 5) return real(map, dtype, rank, base, dims, strides, box, es, il, sw, l2, oob);
    TmaEncodeKey k;
    std::memset(&k, 0, sizeof(k));
    k.base = reinterpret_cast<uint64_t>(base);
    for (cuuint32_t d = 0; d < rank; ++d) {
        k.dims[d] = dims[d];
        k.box[d] = box[d];
        k.es[d] = es[d];
        if (d + 1 < rank) k.strides[d] = strides[d];
    }
    k.dtype = dtype;
    k.rank = rank;
    k.interleave = il;
    k.swizzle = sw;
    k.l2 = l2;
    k.oob = oob;
    uint64_t h = 1469598103934665603ull;  // FNV-1a over the key's bytes
    const unsigned char *kb = reinterpret_cast<const unsigned char *>(&k);
    for (size_t b = 0; b < sizeof(k); ++b) h = (h ^ kb[b]) * 1099511628211ull;
    constexpr int kSlots = 256;
    static std::mutex mu;
    static TmaEncodeKey keys[kSlots];
    static bool used[kSlots];
    static CUtensorMap maps[kSlots];
    const int slot = static_cast<int>(h % kSlots);
    {
        std::lock_guard<std::mutex> lock(mu);
        if (used[slot] && std::memcmp(&keys[slot], &k, sizeof(k)) == 0) {
            *map = maps[slot];
            return CUDA_SUCCESS;
        }
    }
    const CUresult r = real(map, dtype, rank, base, dims, strides, box, es, il, sw, l2, oob);
    if (r == CUDA_SUCCESS) {
        std::lock_guard<std::mutex> lock(mu);
        keys[slot] = k;
        maps[slot] = *map;
        used[slot] = true;
    }
    return r;
}

// The encoder every entry point uses (cached, same contract as the driver's).
inline EncodeTiledFn tma_encode_fn() { return tma_driver_encode_fn() ? &tma_encode_cached : nullptr; }

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
