// Host helper: encode TMA tensor maps (CUtensorMap) for bf16 or 8-bit
// row-major matrices, loaded in boxes whose inner extent is 128 bytes (64
// bf16 or 128 one-byte elements) with the 128-byte swizzle the tcgen05
// shared-memory descriptors expect.
// The driver entry point is fetched through the runtime, so the library
// links only against cudart.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>

namespace moe {

inline PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

inline CUtensorMapDataType tmap_type(unsigned elem_bytes) {
    return elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
}

// rank-2 map over a [rows][cols] matrix of elem_bytes-wide elements (2: bf16,
// 1: an 8-bit format) with row pitch `ld` elements; box = box_cols
// (innermost, 128 bytes) x box_rows.  Out-of-bounds reads fill 0.
inline bool make_tmap_2d(CUtensorMap* m, const void* base, unsigned long long cols, unsigned long long rows,
                         unsigned long long ld, unsigned box_cols, unsigned box_rows, unsigned elem_bytes = 2) {
    auto enc = tmap_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {ld * elem_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t es[2] = {1, 1};
    return enc(m, tmap_type(elem_bytes), 2, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// rank-2 map over `rows` rows of `words` 32-bit words each (contiguous), one
// row per box, no swizzle: the E4M3 scale atoms and token images (512 or
// 1024 bytes), copied as they lie.  Out-of-bounds rows fill 0.
inline bool make_tmap_rows_u32(CUtensorMap* m, const void* base, unsigned words, unsigned long long rows) {
    auto enc = tmap_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {words, rows};
    cuuint64_t strides[1] = {(cuuint64_t)words * 4};
    cuuint32_t box[2] = {words, 1};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// rank-3 fp32 map for tiled stores: [planes][rows][cols] with row pitch
// `ld` and plane pitch `plane` elements; box = box_cols (innermost, 32
// floats = 128 bytes, 128-byte swizzle) x box_rows x 1.
inline bool make_tmap_3d_f32(CUtensorMap* m, void* base, unsigned long long cols, unsigned long long rows,
                             unsigned long long planes, unsigned long long ld, unsigned long long plane,
                             unsigned box_cols, unsigned box_rows) {
    auto enc = tmap_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {cols, rows, planes};
    cuuint64_t strides[2] = {ld * 4, plane * 4};
    cuuint32_t box[3] = {box_cols, box_rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace moe
