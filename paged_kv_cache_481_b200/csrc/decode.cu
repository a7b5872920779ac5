// libpa, decode: C ABI of the paged decode attention (fp16 and int8 caches),
// its workspace, the allocation-free variant, and the device error word.
// Host code here only validates arguments, sizes grids and launches; the
// arithmetic runs in decode_kernel.cuh.  Nothing here allocates device memory.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>

#include "../../include/pa.h"

#include "decode_kernel.cuh"
#include "host_common.cuh"

namespace {

// Workspace: for each worker (warp) two partial-result slots (its first and
// its last (sequence, head), the only ones that can straddle workers), then
// one merge ticket per (sequence, head).
struct WorkspaceLayout {
    size_t o_off, ml_off, count_off, total;
};

WorkspaceLayout workspace_layout(int num_seqs, int num_heads, int head_dim)
{
    WorkspaceLayout w{};
    const size_t units = size_t(num_seqs) * size_t(num_heads);
    const size_t slots = size_t(pa::kMaxWorkers) * 2;
    w.o_off = 0;
    w.ml_off = align256(slots * size_t(head_dim) * sizeof(float));
    w.count_off = w.ml_off + align256(slots * 2 * sizeof(float));
    w.total = w.count_off + align256((units > 0 ? units : 1) * sizeof(unsigned));
    return w;
}

template <int D, bool kInt8, int NW, int S, bool kLateDepWait = false, bool kContig = false>
pa_status launch_decode(const pa::DecodeParams &p, const pa::DecodeExtras &x, cudaStream_t stream,
                        int max_ctas = 0)
{
    using Sm = pa::DecodeSmem<D, kInt8, NW, S>;
    constexpr auto kernel = pa::paged_decode_kernel<D, kInt8, NW, S, kLateDepWait, kContig>;
    static std::atomic<int> grid_for[kMaxDevices];  // 0 = not configured yet
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return PA_ERR_CUDA;
    int grid = grid_for[dev].load(std::memory_order_acquire);
    if (grid == 0) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(Sm::kBytes)) != cudaSuccess)
            return PA_ERR_CUDA;
        int sms = 0, per_sm = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, Sm::kThreads, Sm::kBytes) !=
                cudaSuccess)
            return PA_ERR_CUDA;
        grid = sms * (per_sm > 0 ? per_sm : 1);
        if (grid * NW > pa::kMaxWorkers)
            grid = pa::kMaxWorkers / NW;
        grid_for[dev].store(grid, std::memory_order_release);
    }
    if (max_ctas > 0 && max_ctas < grid)
        grid = max_ctas;
    return launch_pdl(kernel, dim3(grid), dim3(Sm::kThreads), Sm::kBytes, stream, p, x) == cudaSuccess
               ? PA_OK
               : PA_ERR_CUDA;
}

#ifndef PA_DECODE_WARPS
#define PA_DECODE_WARPS 8
#endif
#ifndef PA_DECODE_STAGES
#define PA_DECODE_STAGES 1
#endif
constexpr int kDecodeWarps = PA_DECODE_WARPS;
constexpr int kDecodeStages = PA_DECODE_STAGES;

} // namespace

extern "C" {

pa_status pa_get_last_device_error(unsigned int *code)
{
    if (!code)
        return PA_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess)
        return PA_ERR_CUDA;
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, pa::g_device_error, sizeof(v)) != cudaSuccess)
        return PA_ERR_CUDA;
    if (cudaMemcpyToSymbol(pa::g_device_error, &zero, sizeof(zero)) != cudaSuccess)
        return PA_ERR_CUDA;
    *code = v;
    return PA_OK;
}

} // extern "C"

unsigned int *pa_host::device_error_word()
{
    static std::atomic<void *> addr[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return nullptr;
    void *a = addr[dev].load(std::memory_order_acquire);
    if (!a) {
        if (cudaGetSymbolAddress(&a, pa::g_device_error) != cudaSuccess)
            return nullptr;
        addr[dev].store(a, std::memory_order_release);
    }
    return static_cast<unsigned int *>(a);
}

extern "C" {

size_t pa_decode_workspace_size(int num_seqs, int num_heads, int head_dim, int max_context_len)
{
    if (num_seqs < 0 || num_heads < 0 || head_dim < 0 || max_context_len < 0)
        return 0;
    (void)max_context_len;
    return workspace_layout(num_seqs, num_heads, head_dim).total;
}

pa_status pa_decode_workspace_init(void *workspace, size_t workspace_bytes, pa_stream_t stream)
{
    if (!workspace || workspace_bytes == 0)
        return PA_ERR_INVALID_ARG;
    // The whole workspace is cleared: the counters are all that must start
    // at zero, but zeroing everything keeps the call independent of sizes.
    return cudaMemsetAsync(workspace, 0, workspace_bytes, reinterpret_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? PA_OK
               : PA_ERR_CUDA;
}

} // extern "C"

namespace {

pa_status decode_common(void *out, const void *q, const void *k_cache, const void *v_cache,
                        const void *k_params, const void *v_params, bool int8,
                        const int32_t *block_tables, int max_blocks_per_seq,
                        const int32_t *context_lens, int max_context_len, int num_seqs,
                        int num_heads, int head_dim, int block_size, int num_blocks, float scale,
                        void *workspace, size_t workspace_bytes, pa_stream_t stream,
                        const void *new_k = nullptr, const void *new_v = nullptr,
                        const int64_t *new_slots = nullptr, float *lse = nullptr,
                        int max_ctas = 0, bool late_dep_wait = false,
                        const unsigned int *ready = nullptr)
{
    if (num_seqs < 0 || num_heads <= 0 || num_blocks <= 0 || max_context_len < 0 ||
        max_blocks_per_seq < 0)
        return PA_ERR_INVALID_ARG;
    if (!supported_head_dim(head_dim) || !supported_block_size(block_size))
        return PA_ERR_UNSUPPORTED;
    if (int64_t(max_context_len) > int64_t(max_blocks_per_seq) * block_size)
        return PA_ERR_INVALID_ARG;
    if (!std::isfinite(scale))
        return PA_ERR_INVALID_ARG;
    if (num_seqs == 0)
        return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
        return PA_ERR_INVALID_ARG;
    if (int8 && (!k_params || !v_params || !aligned16(k_params) || !aligned16(v_params)))
        return PA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
        (reinterpret_cast<uintptr_t>(context_lens) & 3u))
        return PA_ERR_INVALID_ARG;
    const WorkspaceLayout w = workspace_layout(num_seqs, num_heads, head_dim);
    if (!workspace || workspace_bytes < w.total || !aligned16(workspace))
        return PA_ERR_WORKSPACE;

    unsigned char *ws = static_cast<unsigned char *>(workspace);
    pa::DecodeParams p{};
    p.out = static_cast<__half *>(out);
    p.q = static_cast<const __half *>(q);
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.k_params = static_cast<const float *>(k_params);
    p.v_params = static_cast<const float *>(v_params);
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.ws_o = reinterpret_cast<float *>(ws + w.o_off);
    p.ws_ml = reinterpret_cast<float *>(ws + w.ml_off);
    p.ws_count = reinterpret_cast<unsigned *>(ws + w.count_off);
    p.num_seqs = num_seqs;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.max_context_len = max_context_len;
    p.num_heads = num_heads;
    p.block_size = block_size;
    p.num_blocks = num_blocks;
    p.qk_scale_log2 = float(double(scale) * 1.4426950408889634);  // scale * log2(e)
    pa::DecodeExtras x{};
    x.new_k = static_cast<const __half *>(new_k);
    x.new_v = static_cast<const __half *>(new_v);
    x.new_slots = new_slots;
    x.lse = lse;
    x.ready = late_dep_wait ? ready : nullptr;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (int8) {
        if (head_dim == 128)
            return launch_decode<128, true, kDecodeWarps, kDecodeStages>(p, x, s);
        return launch_decode<64, true, kDecodeWarps, kDecodeStages>(p, x, s);
    }
    if (late_dep_wait) {
        if (head_dim == 128)
            return launch_decode<128, false, kDecodeWarps, kDecodeStages, true>(p, x, s, max_ctas);
        return launch_decode<64, false, kDecodeWarps, kDecodeStages, true>(p, x, s, max_ctas);
    }
    if (head_dim == 128)
        return launch_decode<128, false, kDecodeWarps, kDecodeStages>(p, x, s, max_ctas);
    return launch_decode<64, false, kDecodeWarps, kDecodeStages>(p, x, s, max_ctas);
}

} // namespace

extern "C" {

pa_status pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                    int max_context_len, int num_seqs, int num_heads, int head_dim, int block_size,
                    int num_blocks, float scale, void *workspace, size_t workspace_bytes,
                    pa_stream_t stream)
{
    return decode_common(out, q, k_cache, v_cache, nullptr, nullptr, false, block_tables,
                         max_blocks_per_seq, context_lens, max_context_len, num_seqs, num_heads,
                         head_dim, block_size, num_blocks, scale, workspace, workspace_bytes, stream);
}

pa_status pa_decode_append(void *out, const void *q, const void *key, const void *value,
                           void *k_cache, void *v_cache, const int64_t *slot_mapping,
                           const int32_t *block_tables, int max_blocks_per_seq,
                           const int32_t *context_lens, int max_context_len, int num_seqs,
                           int num_heads, int head_dim, int block_size, int num_blocks, float scale,
                           void *workspace, size_t workspace_bytes, pa_stream_t stream)
{
    if (num_seqs > 0 && (!key || !value || !slot_mapping || !aligned16(key) || !aligned16(value) ||
                         (reinterpret_cast<uintptr_t>(slot_mapping) & 7u)))
        return PA_ERR_INVALID_ARG;
    return decode_common(out, q, k_cache, v_cache, nullptr, nullptr, false, block_tables,
                         max_blocks_per_seq, context_lens, max_context_len, num_seqs, num_heads,
                         head_dim, block_size, num_blocks, scale, workspace, workspace_bytes, stream,
                         key, value, slot_mapping);
}

pa_status pa_decode_append_int8(void *out, const void *q, const void *key, const void *value,
                                void *k_codes, void *v_codes, void *k_params, void *v_params,
                                const int64_t *slot_mapping, const int32_t *block_tables,
                                int max_blocks_per_seq, const int32_t *context_lens,
                                int max_context_len, int num_seqs, int num_heads, int head_dim,
                                int block_size, int num_blocks, float scale, void *workspace,
                                size_t workspace_bytes, pa_stream_t stream)
{
    if (num_seqs > 0 && (!key || !value || !slot_mapping || !aligned16(key) || !aligned16(value) ||
                         (reinterpret_cast<uintptr_t>(slot_mapping) & 7u)))
        return PA_ERR_INVALID_ARG;
    return decode_common(out, q, k_codes, v_codes, k_params, v_params, true, block_tables,
                         max_blocks_per_seq, context_lens, max_context_len, num_seqs, num_heads,
                         head_dim, block_size, num_blocks, scale, workspace, workspace_bytes, stream,
                         key, value, slot_mapping);
}

pa_status pa_decode_int8(void *out, const void *q, const void *k_codes, const void *v_codes,
                         const void *k_params, const void *v_params, const int32_t *block_tables,
                         int max_blocks_per_seq, const int32_t *context_lens, int max_context_len,
                         int num_seqs, int num_heads, int head_dim, int block_size, int num_blocks,
                         float scale, void *workspace, size_t workspace_bytes, pa_stream_t stream)
{
    return decode_common(out, q, k_codes, v_codes, k_params, v_params, true, block_tables,
                         max_blocks_per_seq, context_lens, max_context_len, num_seqs, num_heads,
                         head_dim, block_size, num_blocks, scale, workspace, workspace_bytes, stream);
}

} // extern "C"

// ---------------------------------------------------------------------------
// The contiguous-cache baseline: the same decode over per-(sequence, head)
// contiguous K / V, [B, H, seq_stride, D], addresses computed from the
// position with no block table.

extern "C" pa_status pa_decode_contiguous(void *out, const void *q, const void *k, const void *v,
                                          const int32_t *context_lens, int max_context_len,
                                          int seq_stride, int num_seqs, int num_heads, int head_dim,
                                          float scale, void *workspace, size_t workspace_bytes,
                                          pa_stream_t stream)
{
    if (num_seqs < 0 || num_heads <= 0 || max_context_len < 0 || seq_stride <= 0 ||
        max_context_len > seq_stride)
        return PA_ERR_INVALID_ARG;
    if (!supported_head_dim(head_dim))
        return PA_ERR_UNSUPPORTED;
    if (!std::isfinite(scale))
        return PA_ERR_INVALID_ARG;
    if (num_seqs == 0)
        return PA_OK;
    if (!out || !q || !k || !v || !context_lens)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
        (reinterpret_cast<uintptr_t>(context_lens) & 3u))
        return PA_ERR_INVALID_ARG;
    const WorkspaceLayout w = workspace_layout(num_seqs, num_heads, head_dim);
    if (!workspace || workspace_bytes < w.total || !aligned16(workspace))
        return PA_ERR_WORKSPACE;
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    pa::DecodeParams p{};
    p.out = static_cast<__half *>(out);
    p.q = static_cast<const __half *>(q);
    p.k_cache = k;
    p.v_cache = v;
    p.block_tables = nullptr;
    p.context_lens = context_lens;
    p.ws_o = reinterpret_cast<float *>(ws + w.o_off);
    p.ws_ml = reinterpret_cast<float *>(ws + w.ml_off);
    p.ws_count = reinterpret_cast<unsigned *>(ws + w.count_off);
    p.num_seqs = num_seqs;
    p.max_blocks_per_seq = 0;
    p.max_context_len = max_context_len;
    p.num_heads = num_heads;
    p.block_size = seq_stride;  // rows per (sequence, head)
    p.num_blocks = num_seqs;
    p.qk_scale_log2 = float(double(scale) * 1.4426950408889634);
    const pa::DecodeExtras x{};
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (head_dim == 128)
        return launch_decode<128, false, kDecodeWarps, kDecodeStages, false, true>(p, x, s);
    return launch_decode<64, false, kDecodeWarps, kDecodeStages, false, true>(p, x, s);
}

// ---------------------------------------------------------------------------
// Allocation-free variant of pa_decode.
//
// Some callers cannot allocate device memory when they call the decode: a
// serving engine typically reserves almost all free HBM for its KV block
// pool at start-up, so a later cudaMalloc for a workspace fails, and
// cudaMalloc/cudaFree can also synchronise the device in the middle of a
// latency-critical decode loop.  For them the split-K workspace lives in the
// file-scope device array below, which the CUDA module reserves on every GPU
// that loads this library and keeps until the process exits.

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB per GPU

// In host code this name is only a host-side stand-in for the array, never a
// device address: kernels get the address from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_no_alloc_scratch[kNoAllocScratchBytes];

std::atomic<void *> g_no_alloc_scratch_addr[kMaxDevices];

// Device address of g_no_alloc_scratch on the current device; looked up once
// per device (with that device current) on the first call there.
pa_status no_alloc_scratch_address(void **addr)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return PA_ERR_CUDA;
    void *p = g_no_alloc_scratch_addr[dev].load(std::memory_order_acquire);
    if (!p) {
        if (cudaGetSymbolAddress(&p, g_no_alloc_scratch) != cudaSuccess || !p)
            return PA_ERR_CUDA;
        g_no_alloc_scratch_addr[dev].store(p, std::memory_order_release);
    }
    *addr = p;
    return PA_OK;
}

} // namespace

extern "C" pa_status pa_decode_no_alloc(void *out, const void *q, const void *k_cache,
                                        const void *v_cache, const int32_t *block_tables,
                                        int max_blocks_per_seq, const int32_t *context_lens,
                                        int max_context_len, int num_seqs, int num_heads,
                                        int head_dim, int block_size, int num_blocks, float scale,
                                        pa_stream_t stream)
{
    if (num_seqs < 0 || num_heads <= 0 || head_dim < 0 || max_context_len < 0)
        return PA_ERR_INVALID_ARG;
    const size_t need = pa_decode_workspace_size(num_seqs, num_heads, head_dim, max_context_len);
    if (need > kNoAllocScratchBytes)
        return PA_ERR_WORKSPACE;  // sizes beyond the static scratch: use pa_decode
    void *scratch = nullptr;
    const pa_status st = no_alloc_scratch_address(&scratch);
    if (st != PA_OK)
        return st;
    // The merge tickets must start at zero; the array keeps whatever the last
    // call (or an aborted one) left there, so clear them on every call.
    if (num_seqs > 0 && supported_head_dim(head_dim)) {
        const WorkspaceLayout w = workspace_layout(num_seqs, num_heads, head_dim);
        if (cudaMemsetAsync(static_cast<unsigned char *>(scratch) + w.count_off, 0,
                            size_t(num_seqs) * size_t(num_heads) * sizeof(unsigned),
                            reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
            return PA_ERR_CUDA;
    }
    return pa_decode(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                     max_context_len, num_seqs, num_heads, head_dim, block_size, num_blocks, scale,
                     scratch, kNoAllocScratchBytes, stream);
}

size_t pa_host::decode_ticket_offset(int num_seqs, int num_heads, int head_dim)
{
    return workspace_layout(num_seqs, num_heads, head_dim).count_off;
}

pa_status pa_host::decode_with_lse(void *out, const void *q, const void *k_cache,
                                   const void *v_cache, const int32_t *block_tables,
                                   int max_blocks_per_seq, const int32_t *context_lens,
                                   int max_context_len, int num_seqs, int num_heads, int head_dim,
                                   int block_size, int num_blocks, float scale, void *workspace,
                                   size_t workspace_bytes, float *lse, pa_stream_t stream,
                                   int max_ctas, bool late_dep_wait, const unsigned int *ready)
{
    return decode_common(out, q, k_cache, v_cache, nullptr, nullptr, false, block_tables,
                         max_blocks_per_seq, context_lens, max_context_len, num_seqs, num_heads,
                         head_dim, block_size, num_blocks, scale, workspace, workspace_bytes, stream,
                         nullptr, nullptr, nullptr, lse, max_ctas, late_dep_wait, ready);
}

int pa_host::decode_ctas_per_sm()
{
    constexpr auto kernel = pa::paged_decode_kernel<128, false, kDecodeWarps, kDecodeStages, true>;
    using Sm = pa::DecodeSmem<128, false, kDecodeWarps, kDecodeStages>;
    int per_sm = 0;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(Sm::kBytes)) !=
            cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, Sm::kThreads, Sm::kBytes) !=
            cudaSuccess)
        return 0;
    return per_sm;
}
