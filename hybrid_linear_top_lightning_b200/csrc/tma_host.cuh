// Host side of TMA: tensor-map encoding through the driver entry point (no
// link-time dependency on libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lisa {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn tma_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2D bf16 tensor of `rows` rows of `inner` elements (row stride inner * 2 bytes),
// boxes of {inner, box_rows}, 128-byte swizzle (inner * 2 must be <= 128).
// Rows past the end read as zero.
inline bool make_tmap_bf16_rows(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                                uint32_t box_rows) {
    EncodeTiledFn fn = tma_encode_fn();
    if (!fn) return false;
    const cuuint64_t gdim[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)inner * 2};
    const cuuint32_t box[2] = {(cuuint32_t)inner, box_rows};
    const cuuint32_t estride[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box,
              estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A 2-D bf16 tensor [rows][inner] read in boxes of box_inner x box_rows with the
// 128-byte swizzle (box_inner * 2 must be 128).
inline bool make_tmap_bf16_box(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                               uint32_t box_inner, uint32_t box_rows) {
    EncodeTiledFn fn = tma_encode_fn();
    if (!fn) return false;
    const cuuint64_t gdim[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)inner * 2};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estride[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box,
              estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A 3-D bf16 tensor [batch][rows][inner] whose rows are `row_stride` elements
// apart and whose batches are `batch_stride` elements apart, read in boxes of
// box_inner (64: 128 bytes) x box_rows x box_batch with the 128-byte swizzle
// (in shared memory: box_rows x box_batch rows of 128 bytes, rows fastest).
// Elements past a dimension's end read as zero.
inline bool make_tmap_bf16_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                              uint64_t batch, uint64_t row_stride, uint64_t batch_stride,
                              uint32_t box_inner, uint32_t box_rows, uint32_t box_batch = 1) {
    EncodeTiledFn fn = tma_encode_fn();
    if (!fn) return false;
    const cuuint64_t gdim[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)batch};
    const cuuint64_t gstride[2] = {(cuuint64_t)row_stride * 2, (cuuint64_t)batch_stride * 2};
    const cuuint32_t box[3] = {box_inner, box_rows, box_batch};
    const cuuint32_t estride[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), gdim, gstride, box,
              estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace lisa
