// tmap.cuh -- TMA tensor-map encoding for the tcgen05 kernels (host side).
//
// The driver's cuTensorMapEncodeTiled is looked up once through the runtime
// (no link against libcuda), and maps are encoded for bf16 or fp32 tensors.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

namespace gqa {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encoder() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// bf16 tensor map with 128-byte swizzle and a {64, rows...} box; OOB reads are zero.
inline bool encode(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims,
                   const cuuint64_t *strides, const cuuint32_t *box) {
    EncodeTiledFn fn = encoder();
    if (!fn) return false;
    cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), dims, strides,
              box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 2-D tensor map [rows][cols] (row stride in bytes a multiple of 16), no
// swizzle, box {box_cols, 1}; OOB reads are zero.
inline bool encode_f32_2d(CUtensorMap *m, const void *base, cuuint64_t cols, cuuint64_t rows,
                          cuuint64_t row_stride_bytes, cuuint32_t box_cols) {
    EncodeTiledFn fn = encoder();
    if (!fn) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {row_stride_bytes};
    const cuuint32_t box[2] = {box_cols, 1};
    cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(base), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace gqa
