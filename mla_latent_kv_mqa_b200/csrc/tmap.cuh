// Host-side TMA tensor-map encoding (driver entry point looked up through the runtime, so the
// library needs no link-time dependency on libcuda).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mla {

inline PFN_cuTensorMapEncodeTiled_v12000 tmap_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2-D map: `rows` rows of `inner` elements, `row_bytes` apart; boxes of box_inner x box_rows with
// 128-byte swizzle (box_inner * element size must be 128).
inline bool tmap_2d(CUtensorMap *m, CUtensorMapDataType dtype, const void *base, uint64_t inner, uint64_t rows,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows) {
    auto fn = tmap_encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    cuuint64_t gstride[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, dtype, 2, const_cast<void *>(base), gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// 3-D bf16 "column-block" map over rows of `cols` elements (`row_bytes` apart): coordinates
// (x in a 64-wide column block, row, column block); a box {64, box_rows, nblk} lands in shared memory
// as nblk consecutive [box_rows x 128 B] tiles with 128-byte swizzle, i.e. the K-major (or MN-major)
// canonical layout of the tensor core, in one TMA operation.
inline bool tmap_bf16_colblocks(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint64_t row_bytes,
                                uint32_t box_rows, uint32_t nblk) {
    auto fn = tmap_encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[3] = {64, (cuuint64_t)rows, (cuuint64_t)(cols / 64)};
    cuuint64_t gstride[2] = {(cuuint64_t)row_bytes, 128};
    cuuint32_t box[3] = {64, box_rows, nblk};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), gdim, gstride, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// 4-D bf16 map over a token-major tensor [rows][heads][cols] (contiguous): coordinates (x in a
// 64-wide column block, row, column block, head); a box {64, box_rows, nblk, 1} lands as nblk
// consecutive [box_rows x 128 B] tiles with 128-byte swizzle: one head's column blocks of
// box_rows consecutive rows, read in place.
inline bool tmap_bf16_head_colblocks(CUtensorMap *m, const void *base, uint64_t rows, uint64_t heads, uint64_t cols,
                                     uint32_t box_rows, uint32_t nblk) {
    auto fn = tmap_encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[4] = {64, (cuuint64_t)rows, (cuuint64_t)(cols / 64), (cuuint64_t)heads};
    cuuint64_t gstride[3] = {(cuuint64_t)(heads * cols * 2), 128, (cuuint64_t)(cols * 2)};
    cuuint32_t box[4] = {64, box_rows, nblk, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), gdim, gstride, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// 2-D byte map without swizzle: boxes of box_inner bytes x box_rows land row-major.
inline bool tmap_u8_rows(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows, uint64_t row_bytes,
                         uint32_t box_inner, uint32_t box_rows) {
    auto fn = tmap_encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    cuuint64_t gstride[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), gdim, gstride, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// 3-D byte "column-block" map over rows of `cols` bytes (`row_bytes` apart): coordinates
// (x in a 128-byte column block, row, column block); a box {128, box_rows, nblk} lands as nblk
// consecutive [box_rows x 128 B] tiles with 128-byte swizzle (the K-major layout of 8-bit
// tensor-core operands).
inline bool tmap_u8_colblocks(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint64_t row_bytes,
                              uint32_t box_rows, uint32_t nblk) {
    auto fn = tmap_encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[3] = {128, (cuuint64_t)rows, (cuuint64_t)(cols / 128)};
    cuuint64_t gstride[2] = {(cuuint64_t)row_bytes, 128};
    cuuint32_t box[3] = {128, box_rows, nblk};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), gdim, gstride, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
inline bool tmap_bf16_2d(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows, uint64_t row_bytes,
                         uint32_t box_inner, uint32_t box_rows) {
    return tmap_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, inner, rows, row_bytes, box_inner, box_rows);
}

}  // namespace mla
