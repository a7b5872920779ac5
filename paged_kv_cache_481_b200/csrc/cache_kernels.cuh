// Cache write (slot scatter) and copy-on-write block copy for sm_100a.
// Both are pure data movement with 16-byte vector accesses; bit-exact.
#pragma once

#include <cstdint>

#include "decode_kernel.cuh"  // g_device_error / raise_device_error

namespace pa {

// polomodov.tech "vLLM and PagedAttention", slide 11: each new token goes into
// the next free slot of its sequence's last block.  Grid (num_tokens, 2): y = 0
// writes K, y = 1 writes V.  A token's H*D row is contiguous in the input; in
// the cache its heads sit block_size*D elements apart.
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(
    const uint4 *__restrict__ key, const uint4 *__restrict__ value, uint4 *__restrict__ k_cache,
    uint4 *__restrict__ v_cache, const int64_t *__restrict__ slot_mapping, int num_heads,
    int head_chunks, int block_size, int num_blocks)
{
    grid_dependency_wait();
    allow_dependent_launch();
    const int i = blockIdx.x;
    const int64_t slot = slot_mapping[i];
    if (slot < 0)
        return;
    if (slot >= int64_t(num_blocks) * block_size) {
        if (threadIdx.x == 0 && blockIdx.y == 0)
            raise_device_error(1u << 2);
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

// comfyai.app "6.4 PagedAttention", 6.4.2-6.4.3 / polomodov.tech slide 13:
// copy-on-write duplicates a shared block before a divergent write.  Grid
// (num_pairs, 2, chunks): y selects K or V, z a 16 KB chunk of the block.
constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 4;

__global__ void __launch_bounds__(kCopyThreads) copy_blocks_kernel(
    uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache, const int64_t *__restrict__ block_mapping,
    int64_t block_vecs, int num_blocks)
{
    grid_dependency_wait();
    allow_dependent_launch();
    const int pair = blockIdx.x;
    const int64_t src = block_mapping[2 * pair], dst = block_mapping[2 * pair + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
        if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
            raise_device_error(1u << 3);
        return;
    }
    uint4 *cache = blockIdx.y == 0 ? k_cache : v_cache;
    const uint4 *s = cache + src * block_vecs;
    uint4 *d = cache + dst * block_vecs;
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
__global__ void __launch_bounds__(32) bounded_wait_selftest_kernel(uint64_t limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        fence_mbar_init();
    }
    __syncwarp();
    const bool ok = mbar_wait_bounded(smem_u32(&bar), 0u, limit_ns);
    if (!__all_sync(kFullMask, ok) && threadIdx.x == 0)
        raise_device_error(kErrTimeout);
}

} // namespace pa
