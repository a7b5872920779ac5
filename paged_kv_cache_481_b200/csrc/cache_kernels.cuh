// Cache writes (slot scatter, fp16 and int8), whole-block copies and the
// bounded-wait self-test for sm_100a.  Errors are OR-ed into the device error
// word `err` (PA_DEVERR_* bits).
#pragma once

#include <cuda_fp16.h>

#include <cstdint>

#include "../../include/pa.h"
#include "ptx.cuh"
#include "quant.cuh"

namespace pa {

// polomodov.tech "vLLM and PagedAttention", slide 11: each new token goes into
// the next free slot of its sequence's last block.  Grid (num_tokens, 2): y = 0
// writes K, y = 1 writes V.  A token's H*D row is contiguous in the input; in
// the cache its heads sit block_size*D elements apart.
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(
    const uint4 *__restrict__ key, const uint4 *__restrict__ value, uint4 *__restrict__ k_cache,
    uint4 *__restrict__ v_cache, const int64_t *__restrict__ slot_mapping, int num_heads,
    int head_chunks, int block_size, int num_blocks, unsigned int *err)
{
    grid_dependency_wait();
    allow_dependent_launch();
    const int i = blockIdx.x;
    const int64_t slot = slot_mapping[i];
    if (slot < 0)
        return;
    if (slot >= int64_t(num_blocks) * block_size) {
        if (threadIdx.x == 0 && blockIdx.y == 0)
            atomicOr(err, PA_DEVERR_SLOT);
        return;
    }
    const int64_t block = slot / block_size, offset = slot % block_size;
    const int n = num_heads * head_chunks;
    const uint4 *src = (blockIdx.y == 0 ? key : value) + int64_t(i) * n;
    uint4 *dst = (blockIdx.y == 0 ? k_cache : v_cache) +
                 (block * num_heads * block_size + offset) * head_chunks;
    const int64_t head_stride = int64_t(block_size) * head_chunks;
    for (int e = threadIdx.x; e < n; e += blockDim.x) {
        const int hh = e / head_chunks, cc = e - hh * head_chunks;
        dst[hh * head_stride + cc] = __ldg(src + e);
    }
}

// Cache write into the int8 cache (brentwoodlivery.com 5.3.18: affine
// quantization with one (s, z) per group, here per (token, head) row of D
// values, b = 8; quantize_row_warp).  One warp per (token, head) row; grid
// (num_tokens, ceil(H / 4), 2): z = 0 writes K, 1 writes V.
template <int D>
__global__ void __launch_bounds__(128) reshape_and_cache_int8_kernel(
    const __half *__restrict__ key, const __half *__restrict__ value, uint8_t *__restrict__ k_codes,
    uint8_t *__restrict__ v_codes, float2 *__restrict__ k_params, float2 *__restrict__ v_params,
    const int64_t *__restrict__ slot_mapping, int num_heads, int block_size, int num_blocks,
    unsigned int *err)
{
    grid_dependency_wait();
    allow_dependent_launch();
    constexpr int E = D / 32;  // values per lane
    const int i = blockIdx.x, lane = threadIdx.x & 31;
    const int h = blockIdx.y * 4 + (threadIdx.x >> 5);
    if (h >= num_heads)
        return;
    const int64_t slot = slot_mapping[i];
    if (slot < 0)
        return;
    if (slot >= int64_t(num_blocks) * block_size) {
        if (lane == 0 && h == 0 && blockIdx.z == 0)
            atomicOr(err, PA_DEVERR_SLOT);
        return;
    }
    const bool is_v = blockIdx.z == 1;
    const __half *src = (is_v ? value : key) + (size_t(i) * num_heads + h) * D + lane * E;
    float x[E];
#pragma unroll
    for (int e = 0; e < E; ++e)
        x[e] = __half2float(src[e]);
    float sc, z;
    const uint32_t packed = quantize_row_warp<E>(x, sc, z);
    const int64_t row = (slot / block_size) * num_heads * block_size + int64_t(h) * block_size +
                        slot % block_size;
    uint8_t *dst = (is_v ? v_codes : k_codes) + row * D + lane * E;
    if constexpr (E == 4)
        *reinterpret_cast<uint32_t *>(dst) = packed;
    else
        *reinterpret_cast<uint16_t *>(dst) = uint16_t(packed);
    if (lane == 0)
        (is_v ? v_params : k_params)[row] = make_float2(sc, z);
}

// Whole-block copies.  comfyai.app "6.4 PagedAttention", 6.4.2-6.4.3 /
// polomodov.tech slide 13: copy-on-write duplicates a shared block inside a
// pool before a divergent write; slide 15: a preempted request's blocks are
// swapped between the device pool and a pool in host memory.  Pair i copies
// block map[2i] of the source pool to block map[2i+1] of the destination pool.
// Grid (num_pairs, pools, chunks): y selects the (src, dst) pool pair (K or
// V), z a 16 KB chunk of the block.
constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 4;

__global__ void __launch_bounds__(kCopyThreads) copy_blocks_kernel(
    const uint4 *src0, uint4 *dst0, const uint4 *src1, uint4 *dst1,
    const int64_t *__restrict__ block_mapping, int64_t block_vecs, int num_src_blocks,
    int num_dst_blocks, unsigned int *err)
{
    grid_dependency_wait();
    allow_dependent_launch();
    const int pair = blockIdx.x;
    const int64_t src = block_mapping[2 * pair], dst = block_mapping[2 * pair + 1];
    if (src < 0 || src >= num_src_blocks || dst < 0 || dst >= num_dst_blocks) {
        if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
            atomicOr(err, PA_DEVERR_COPY_PAIR);
        return;
    }
    const uint4 *s = (blockIdx.y == 0 ? src0 : src1) + src * block_vecs;
    uint4 *d = (blockIdx.y == 0 ? dst0 : dst1) + dst * block_vecs;
    const int64_t base = int64_t(blockIdx.z) * kCopyThreads * kCopyUnroll + threadIdx.x;
    uint4 tmp[kCopyUnroll];
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
        const int64_t idx = base + int64_t(u) * kCopyThreads;
        if (idx < block_vecs)
            tmp[u] = __ldcs(s + idx);
    }
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
        const int64_t idx = base + int64_t(u) * kCopyThreads;
        if (idx < block_vecs)
            __stcs(d + idx, tmp[u]);
    }
}

// Self-test of the bounded wait every kernel here relies on: one warp waits
// on an mbarrier that nothing ever arrives at; the wait must give up after
// limit_ns and record PA_DEVERR_TIMEOUT, leaving the context usable.
__global__ void __launch_bounds__(32) bounded_wait_selftest_kernel(uint64_t limit_ns, unsigned int *err)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        fence_mbar_init();
    }
    __syncwarp();
    const bool ok = mbar_wait_bounded(smem_u32(&bar), 0u, limit_ns);
    if (!__all_sync(kFullMask, ok) && threadIdx.x == 0)
        atomicOr(err, PA_DEVERR_TIMEOUT);
}

} // namespace pa
