// libpa, multi-query attention: C ABI of the tensor-core prefill /
// chunked-prefill kernel.  Host code here only validates arguments, encodes
// the TMA tensor maps and launches; the arithmetic runs in
// prefill_kernel.cuh.  Nothing here allocates device memory.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>

#include "../../include/pa.h"
#include "host_common.cuh"
#include "prefill_kernel.cuh"
#include "tma_host.cuh"

namespace {

// Work counters of the persistent prefill kernel: each launch takes the next
// of kSchedSlots (next item, CTAs finished) pairs, which start at zero (module
// load) and are reset by the launch's last CTA.  Slots rotate per device, so
// launches on different streams get different counters as long as fewer than
// kSchedSlots prefill launches are in flight on a device at once.
constexpr int kSchedSlots = 64;
__device__ unsigned int g_prefill_sched[kSchedSlots][2];

unsigned int *next_sched_slot(int dev)
{
    static std::atomic<void *> base[kMaxDevices];
    static std::atomic<unsigned> turn[kMaxDevices];
    void *b = base[dev].load(std::memory_order_acquire);
    if (!b) {
        if (cudaGetSymbolAddress(&b, g_prefill_sched) != cudaSuccess || !b)
            return nullptr;
        base[dev].store(b, std::memory_order_release);
    }
    const unsigned slot = turn[dev].fetch_add(1u, std::memory_order_relaxed) % kSchedSlots;
    return static_cast<unsigned int *>(b) + 2 * slot;
}

// Encode the tensor maps and launch the persistent kernel (arguments already
// validated).
pa_status launch_prefill(void *out, const void *q, const void *k_cache, const void *v_cache,
                         const int32_t *block_tables, int max_blocks_per_seq,
                         const int32_t *context_lens, int max_context_len,
                         const int32_t *query_start_loc, int num_tokens, int max_query_len,
                         int num_seqs, int num_heads, int head_dim, int block_size, int num_blocks,
                         float scale, cudaStream_t stream)
{
    CUtensorMap tm_q, tm_k, tm_v;
    const uint64_t cache_rows = uint64_t(num_blocks) * num_heads * block_size;
    const uint32_t box_rows = uint32_t(block_size < pa::kPN ? block_size : pa::kPN);
    if (!make_map(&tm_q, q, uint64_t(num_heads) * head_dim, uint64_t(num_tokens),
                  uint64_t(num_heads) * head_dim * 2, pa::kPM) ||
        !make_map(&tm_k, k_cache, head_dim, cache_rows, uint64_t(head_dim) * 2, box_rows) ||
        !make_map(&tm_v, v_cache, head_dim, cache_rows, uint64_t(head_dim) * 2, box_rows))
        return PA_ERR_CUDA;

    static std::atomic<int> sm_count[kMaxDevices];  // 0 = not configured yet
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return PA_ERR_CUDA;
    int sms = sm_count[dev].load(std::memory_order_acquire);
    if (sms == 0) {
        if (cudaFuncSetAttribute(pa::paged_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(pa::kPrefillSmem)) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            sms <= 0)
            return PA_ERR_CUDA;
        sm_count[dev].store(sms, std::memory_order_release);
    }
    pa::PrefillParams p{};
    p.out = static_cast<__half *>(out);
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.query_start_loc = query_start_loc;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.max_context_len = max_context_len;
    p.num_heads = num_heads;
    p.block_size = block_size;
    p.num_blocks = num_blocks;
    p.error_word = device_error_word();
    if (!p.error_word)
        return PA_ERR_CUDA;
    p.qk_scale_log2 = float(double(scale) * 1.4426950408889634);
    p.num_rows = num_tokens;
    // persistent: one CTA per SM (the shared-memory footprint allows one),
    // never more CTAs than items
    constexpr int kRowsPerItem = pa::kQTiles * pa::kPM;
    p.num_seqs = num_seqs;
    p.num_pairs = (max_query_len + kRowsPerItem - 1) / kRowsPerItem;
    const int64_t items = int64_t(p.num_pairs) * num_heads * num_seqs;
    if (items > (int64_t(1) << 30))
        return PA_ERR_INVALID_ARG;
    p.sched = next_sched_slot(dev);
    if (!p.sched)
        return PA_ERR_CUDA;
    const dim3 grid(unsigned(items < sms ? items : sms));
    return launch_pdl(pa::paged_prefill_kernel, grid, dim3(pa::kPrefillThreads), pa::kPrefillSmem,
                      stream, tm_q, tm_k, tm_v, p) == cudaSuccess
               ? PA_OK
               : PA_ERR_CUDA;
}

} // namespace

extern "C" pa_status pa_prefill(void *out, const void *q, const void *k_cache, const void *v_cache,
                                const int32_t *block_tables, int max_blocks_per_seq,
                                const int32_t *context_lens, int max_context_len,
                                const int32_t *query_start_loc, int num_tokens, int max_query_len,
                                int num_seqs, int num_heads, int head_dim, int block_size,
                                int num_blocks, float scale, pa_stream_t stream)
{
    if (num_seqs < 0 || num_tokens < 0 || max_query_len < 0 || num_heads <= 0 || num_blocks <= 0 ||
        max_context_len < 0 || max_blocks_per_seq < 0)
        return PA_ERR_INVALID_ARG;
    if (head_dim != pa::kPD || !supported_block_size(block_size))
        return PA_ERR_UNSUPPORTED;
    if (int64_t(max_context_len) > int64_t(max_blocks_per_seq) * block_size ||
        max_query_len > max_context_len || !std::isfinite(scale) || !(scale > 0.f))
        return PA_ERR_INVALID_ARG;
    if (num_seqs == 0 || num_tokens == 0 || max_query_len == 0)
        return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start_loc)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
        (reinterpret_cast<uintptr_t>(context_lens) & 3u) ||
        (reinterpret_cast<uintptr_t>(query_start_loc) & 3u))
        return PA_ERR_INVALID_ARG;
    if (num_seqs > 65535 || num_heads > 65535 ||
        int64_t(num_blocks) * num_heads * block_size > INT32_MAX)
        return PA_ERR_INVALID_ARG;
    return launch_prefill(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                          max_context_len, query_start_loc, num_tokens, max_query_len, num_seqs,
                          num_heads, head_dim, block_size, num_blocks, scale,
                          reinterpret_cast<cudaStream_t>(stream));
}
