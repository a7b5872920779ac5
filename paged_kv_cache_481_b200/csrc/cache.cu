// libpa, cache maintenance: C ABI of the cache writes (fp16 and int8),
// copy-on-write block copies, block swaps between pools, the bounded-wait
// self-test and the status strings.  Host code here only validates
// arguments and launches the kernels of cache_kernels.cuh.  Nothing here
// allocates device memory.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/pa.h"
#include "cache_kernels.cuh"
#include "host_common.cuh"

namespace {

// True if a kernel on the current device may dereference `p` as is: device
// or managed memory, or page-locked host memory mapped at the same address.
// Pageable host memory (which a kernel cannot touch) is refused here.
bool device_addressable(const void *p)
{
    if (!p)
        return false;
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();  // clear the (non-sticky) error the query recorded
        return false;
    }
    switch (a.type) {
    case cudaMemoryTypeDevice:
    case cudaMemoryTypeManaged:
        return true;
    case cudaMemoryTypeHost:
        return a.devicePointer == p;
    default:
        return false;
    }
}

// One pool array's blocks from `src` to `dst` (the same array for
// copy-on-write, or a device and a host pool for swapping).
pa_status launch_block_copies(const void *src, void *dst, size_t block_bytes,
                              const int64_t *block_mapping, int num_pairs, int num_src_blocks,
                              int num_dst_blocks, pa_stream_t stream)
{
    if (num_pairs < 0 || num_src_blocks <= 0 || num_dst_blocks <= 0 || block_bytes == 0 ||
        (block_bytes & 15u))
        return PA_ERR_INVALID_ARG;
    if (num_pairs == 0)
        return PA_OK;
    if (!src || !dst || !block_mapping || !aligned16(src) || !aligned16(dst) ||
        (reinterpret_cast<uintptr_t>(block_mapping) & 7u))
        return PA_ERR_INVALID_ARG;
    const int64_t block_vecs = int64_t(block_bytes / 16);
    const int64_t per_cta = int64_t(pa::kCopyThreads) * pa::kCopyUnroll;
    const int64_t chunks = (block_vecs + per_cta - 1) / per_cta;
    if (chunks > 65535)
        return PA_ERR_INVALID_ARG;
    unsigned int *err = device_error_word();
    if (!err)
        return PA_ERR_CUDA;
    const dim3 grid(unsigned(num_pairs), 1, unsigned(chunks));
    const uint4 *s = static_cast<const uint4 *>(src);
    uint4 *d = static_cast<uint4 *>(dst);
    return launch_pdl(pa::copy_blocks_kernel, grid, dim3(pa::kCopyThreads), 0,
                      reinterpret_cast<cudaStream_t>(stream), s, d, s, d, block_mapping,
                      block_vecs, num_src_blocks, num_dst_blocks, err) == cudaSuccess
               ? PA_OK
               : PA_ERR_CUDA;
}

} // namespace

extern "C" {

pa_status pa_copy_blocks_raw(void *cache, size_t block_bytes, const int64_t *block_mapping,
                             int num_pairs, int num_blocks, pa_stream_t stream)
{
    return launch_block_copies(cache, cache, block_bytes, block_mapping, num_pairs, num_blocks,
                               num_blocks, stream);
}

pa_status pa_swap_blocks(const void *src, void *dst, size_t block_bytes,
                         const int64_t *block_mapping, int num_pairs, int num_src_blocks,
                         int num_dst_blocks, pa_stream_t stream)
{
    if (src == dst && src != nullptr)
        return PA_ERR_INVALID_ARG;  // within one pool: pa_copy_blocks_raw
    if (num_pairs > 0 && (!device_addressable(src) || !device_addressable(dst) ||
                          !device_addressable(block_mapping)))
        return PA_ERR_INVALID_ARG;
    return launch_block_copies(src, dst, block_bytes, block_mapping, num_pairs, num_src_blocks,
                               num_dst_blocks, stream);
}


const char *pa_status_string(pa_status status)
{
    switch (status) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID_ARG: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported head_dim or block_size";
    case PA_ERR_CUDA: return "CUDA runtime error";
    case PA_ERR_WORKSPACE: return "workspace missing or too small";
    case PA_ERR_OUT_OF_BLOCKS: return "no free blocks left in the pool";
    }
    return "unknown status";
}

pa_status pa_reshape_and_cache(const void *key, const void *value, void *k_cache, void *v_cache,
                               const int64_t *slot_mapping, int num_tokens, int num_heads,
                               int head_dim, int block_size, int num_blocks, pa_stream_t stream)
{
    if (num_tokens < 0 || num_heads <= 0 || num_blocks <= 0)
        return PA_ERR_INVALID_ARG;
    if (!supported_head_dim(head_dim) || !supported_block_size(block_size))
        return PA_ERR_UNSUPPORTED;
    if (num_tokens == 0)
        return PA_OK;
    if (!key || !value || !k_cache || !v_cache || !slot_mapping)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
        return PA_ERR_INVALID_ARG;
    unsigned int *err = device_error_word();
    if (!err)
        return PA_ERR_CUDA;
    const dim3 grid(unsigned(num_tokens), 2);
    return launch_pdl(pa::reshape_and_cache_kernel, grid, dim3(128), 0,
                      reinterpret_cast<cudaStream_t>(stream), static_cast<const uint4 *>(key),
                      static_cast<const uint4 *>(value), static_cast<uint4 *>(k_cache),
                      static_cast<uint4 *>(v_cache), slot_mapping, num_heads, head_dim / 8,
                      block_size, num_blocks, err) == cudaSuccess
               ? PA_OK
               : PA_ERR_CUDA;
}

pa_status pa_reshape_and_cache_int8(const void *key, const void *value, void *k_codes,
                                    void *v_codes, void *k_params, void *v_params,
                                    const int64_t *slot_mapping, int num_tokens, int num_heads,
                                    int head_dim, int block_size, int num_blocks, pa_stream_t stream)
{
    if (num_tokens < 0 || num_heads <= 0 || num_blocks <= 0)
        return PA_ERR_INVALID_ARG;
    if (!supported_head_dim(head_dim) || !supported_block_size(block_size))
        return PA_ERR_UNSUPPORTED;
    if (num_tokens == 0)
        return PA_OK;
    if (!key || !value || !k_codes || !v_codes || !k_params || !v_params || !slot_mapping)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(key) || !aligned16(value) || !aligned16(k_codes) || !aligned16(v_codes) ||
        !aligned16(k_params) || !aligned16(v_params) ||
        (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
        return PA_ERR_INVALID_ARG;
    unsigned int *err = device_error_word();
    if (!err)
        return PA_ERR_CUDA;
    const dim3 grid(unsigned(num_tokens), unsigned((num_heads + 3) / 4), 2);
    cudaError_t e;
    if (head_dim == 128)
        e = launch_pdl(pa::reshape_and_cache_int8_kernel<128>, grid, dim3(128), 0,
                       reinterpret_cast<cudaStream_t>(stream), static_cast<const __half *>(key),
                       static_cast<const __half *>(value), static_cast<uint8_t *>(k_codes),
                       static_cast<uint8_t *>(v_codes), static_cast<float2 *>(k_params),
                       static_cast<float2 *>(v_params), slot_mapping, num_heads, block_size,
                       num_blocks, err);
    else
        e = launch_pdl(pa::reshape_and_cache_int8_kernel<64>, grid, dim3(128), 0,
                       reinterpret_cast<cudaStream_t>(stream), static_cast<const __half *>(key),
                       static_cast<const __half *>(value), static_cast<uint8_t *>(k_codes),
                       static_cast<uint8_t *>(v_codes), static_cast<float2 *>(k_params),
                       static_cast<float2 *>(v_params), slot_mapping, num_heads, block_size,
                       num_blocks, err);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_selftest_bounded_wait(unsigned int limit_us, pa_stream_t stream)
{
    if (limit_us == 0 || limit_us > 2000000u)
        return PA_ERR_INVALID_ARG;
    unsigned int *err = device_error_word();
    if (!err)
        return PA_ERR_CUDA;
    pa::bounded_wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        uint64_t(limit_us) * 1000ull, err);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_copy_blocks(void *k_cache, void *v_cache, const int64_t *block_mapping, int num_pairs,
                         int num_heads, int head_dim, int block_size, int num_blocks,
                         pa_stream_t stream)
{
    if (num_pairs < 0 || num_heads <= 0 || num_blocks <= 0)
        return PA_ERR_INVALID_ARG;
    if (!supported_head_dim(head_dim) || !supported_block_size(block_size))
        return PA_ERR_UNSUPPORTED;
    if (num_pairs == 0)
        return PA_OK;
    if (!k_cache || !v_cache || !block_mapping)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(k_cache) || !aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(block_mapping) & 7u))
        return PA_ERR_INVALID_ARG;
    const int64_t block_vecs = int64_t(num_heads) * block_size * head_dim / 8;
    const int64_t per_cta = int64_t(pa::kCopyThreads) * pa::kCopyUnroll;
    const int64_t chunks = (block_vecs + per_cta - 1) / per_cta;
    if (chunks > 65535)
        return PA_ERR_INVALID_ARG;
    unsigned int *err = device_error_word();
    if (!err)
        return PA_ERR_CUDA;
    const dim3 grid(unsigned(num_pairs), 2, unsigned(chunks));
    uint4 *k = static_cast<uint4 *>(k_cache), *v = static_cast<uint4 *>(v_cache);
    return launch_pdl(pa::copy_blocks_kernel, grid, dim3(pa::kCopyThreads), 0,
                      reinterpret_cast<cudaStream_t>(stream), k, k, v, v, block_mapping, block_vecs,
                      num_blocks, num_blocks, err) == cudaSuccess
               ? PA_OK
               : PA_ERR_CUDA;
}

} // extern "C"
