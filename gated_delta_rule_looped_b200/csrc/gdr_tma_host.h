// gdr_tma_host.h -- host-side TMA tensor maps of the [units][L][128] bf16 tensors (q, k, v, o)
// used by the tensor-core prefills.  The driver's encoder is fetched once through the runtime
// (no link against libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

namespace lt2 {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn tma_encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

// 3-D view [units][L][128] of a bf16 tensor with boxes of 64 columns x `box_rows` tokens x 1
// unit.  Rows past a unit's L are zero-filled on loads and dropped on stores, so a box never
// touches the next unit.  Every coordinate the kernels use on the column axis is 0 or 64
// (128-byte aligned), and the row stride is 256 bytes.
inline bool make_bf16_map_3d(CUtensorMap* m, const void* base, int64_t units, int64_t L, uint32_t box_rows,
                             CUtensorMapSwizzle swizzle)
{
    EncodeTiledFn fn = tma_encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(units)};
    const cuuint64_t strides[2] = {128 * 2, static_cast<cuuint64_t>(L) * 128 * 2};
    const cuuint32_t box[3] = {64, box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D view [units][L][128] of an fp32 tensor (per-key gates), boxes of all 128 columns x
// `box_rows` tokens x 1 unit, no swizzle (a 512-byte row per token).
inline bool make_f32_map_3d(CUtensorMap* m, const void* base, int64_t units, int64_t L, uint32_t box_rows)
{
    EncodeTiledFn fn = tma_encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(units)};
    const cuuint64_t strides[2] = {128 * 4, static_cast<cuuint64_t>(L) * 128 * 4};
    const cuuint32_t box[3] = {128, box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace lt2
