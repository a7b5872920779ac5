// Host side of the TMA tensor loads: the driver's tensor-map encoder (looked
// up once through the runtime) and 2-D fp16 maps with 128-byte swizzle.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdint>

namespace {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static std::atomic<void *> fn{nullptr};
    void *f = fn.load(std::memory_order_acquire);
    if (!f) {
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn.store(f, std::memory_order_release);
    }
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
}

// 2-D fp16 tensor map with 128-byte swizzle: `rows` rows of `cols` elements,
// `row_bytes` apart, read in boxes of 64 x box_rows.
bool make_map(CUtensorMap *map, const void *base, uint64_t cols, uint64_t rows, uint64_t row_bytes,
              uint32_t box_rows)
{
    auto encode = tensor_map_encoder();
    if (!encode)
        return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t elem[2] = {1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides,
                  box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

} // namespace

namespace {

// K / V cache rows (256 bytes: 128 fp16) as a 4-D fp16 tensor map with
// 128-byte swizzle whose box is one whole run of `box_rows` rows (a multiple
// of 8): dims (64 elements of a half row; 8 rows of a group, 256 B apart; the
// two 64-element halves, 128 B apart; groups of 8 rows, 2048 B apart).  The
// box lands in shared memory as [row group][half][8 rows][128 B], i.e. each
// (row group, half) is one 1 KB swizzle atom.
bool make_kv_map(CUtensorMap *map, const void *base, uint64_t rows, uint32_t box_rows)
{
    auto encode = tensor_map_encoder();
    if (!encode || rows % 8 != 0 || box_rows % 8 != 0)
        return false;
    const cuuint64_t dims[4] = {64, 8, 2, rows / 8};
    const cuuint64_t strides[3] = {256, 128, 2048};
    const cuuint32_t box[4] = {64, 8, 2, box_rows / 8};
    const cuuint32_t elem[4] = {1, 1, 1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void *>(base), dims, strides,
                  box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

} // namespace
