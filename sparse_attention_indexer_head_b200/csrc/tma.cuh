// TMA tensor maps (host) and 2-D tiled TMA loads (device).
//
// The encoder, cuTensorMapEncodeTiled, is a driver-API entry point; it is
// fetched once through cudaGetDriverEntryPoint so the library needs no link
// against libcuda. Only the CUtensorMap type and enums come from <cuda.h>.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace dsa {

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (EncodeTiledFn) nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// Row-major bf16 matrix [rows, cols] (row stride in bytes), boxes of
// box_cols x box_rows elements landing in shared memory with the 128-byte
// swizzle. Rows outside [0, rows) read as zero.
inline bool make_map_bf16_2d(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols,
                             uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows) {
    const EncodeTiledFn fn = encode_tiled();
    if (!fn || rows == 0) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {row_stride_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t elem[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
              elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tiled 2-D load of the box at element coordinates (x = column, y = row) into
// shared memory at dst, completing on bar through the transaction count. x is
// a multiple of 64 elements (128 bytes) at every call site.
DSA_DEVINL void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

}  // namespace dsa
