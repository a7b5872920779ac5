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
// validated).  grouped / o_f32 / lse: see PrefillParams.
pa_status launch_prefill(void *out, const void *q, const void *k_cache, const void *v_cache,
                         const int32_t *block_tables, int max_blocks_per_seq,
                         const int32_t *context_lens, int max_context_len,
                         const int32_t *query_start_loc, int num_tokens, int max_query_len,
                         int num_seqs, int num_heads, int head_dim, int block_size, int num_blocks,
                         float scale, bool grouped, float *o_f32, float *lse, cudaStream_t stream)
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
    p.grouped = grouped ? 1 : 0;
    p.num_rows = num_tokens;
    p.o_f32 = o_f32;
    p.lse = lse;
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

// ---- shared-prefix (grouped) decode ---------------------------------------

// For member m of group g (block (g, m)): its tail table (its block-table row
// from the first block past the shared prefix on, padded with -1), its tail
// length L_b - P_g, and P_g.  A prefix that is not a whole number of blocks,
// or longer than this member's context, is recorded (PA_DEVERR_CONTEXT_LEN)
// and treated as empty for this member.
__global__ void __launch_bounds__(128) grouped_tails_kernel(
    const int32_t *__restrict__ block_tables, int max_blocks, const int32_t *__restrict__ context_lens,
    int max_context_len, const int32_t *__restrict__ group_start,
    const int32_t *__restrict__ prefix_lens, int block_size, int num_seqs,
    int32_t *__restrict__ tail_tables, int32_t *__restrict__ tail_lens,
    int32_t *__restrict__ prefix_of, unsigned int *err)
{
    pa::grid_dependency_wait();
    pa::allow_dependent_launch();
    const int g = blockIdx.x;
    const int b0 = group_start[g], b1 = group_start[g + 1];
    const int b = b0 + int(blockIdx.y);
    if (b0 < 0 || b1 < b0 || b1 > num_seqs) {  // group bounds outside the batch
        if (threadIdx.x == 0 && blockIdx.y == 0)
            atomicOr(err, PA_DEVERR_CONTEXT_LEN);
        return;
    }
    if (b >= b1)
        return;
    const int L = max(0, min(context_lens[b], max_context_len));
    int P = prefix_lens[g];
    if (P < 0 || P % block_size != 0 || P > L) {
        if (threadIdx.x == 0)
            atomicOr(err, PA_DEVERR_CONTEXT_LEN);
        P = 0;
    }
    const int pb = P / block_size;
    const int32_t *row = block_tables + size_t(b) * max_blocks;
    int32_t *trow = tail_tables + size_t(b) * max_blocks;
    for (int k = threadIdx.x; k < max_blocks; k += blockDim.x)
        trow[k] = pb + k < max_blocks ? row[pb + k] : -1;
    if (threadIdx.x == 0) {
        tail_lens[b] = L - P;
        prefix_of[b] = P;
    }
}

// out = the softmax-weighted combination of the prefix part (fp32, its
// base-2 log-normaliser lse_p) and the tail part (fp16, lse_t): with
// M = max(lse_p, lse_t), out = (2^(lse_p - M) o_p + 2^(lse_t - M) o_t) /
// (2^(lse_p - M) + 2^(lse_t - M)); an empty part has weight 0.  One warp per
// (sequence, head), four dims per lane (D = 128).
__global__ void __launch_bounds__(256) grouped_merge_kernel(
    __half *__restrict__ out, const float *__restrict__ o_p, const float *__restrict__ lse_p,
    const __half *__restrict__ o_t, const float *__restrict__ lse_t,
    const int32_t *__restrict__ prefix_of, const int32_t *__restrict__ tail_lens, int num_heads,
    int units)
{
    pa::grid_dependency_wait();
    pa::allow_dependent_launch();
    const int unit = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (unit >= units)
        return;
    const int b = unit / num_heads;
    const bool has_p = prefix_of[b] > 0, has_t = tail_lens[b] > 0;
    const float lp = has_p ? lse_p[unit] : -INFINITY, lt = has_t ? lse_t[unit] : -INFINITY;
    const float M = fmaxf(lp, lt);
    const float wp = has_p ? exp2f(lp - M) : 0.f, wt = has_t ? exp2f(lt - M) : 0.f;
    const float inv = 1.f / (wp + wt);
    const float4 a = has_p ? reinterpret_cast<const float4 *>(o_p + size_t(unit) * 128)[lane]
                           : make_float4(0.f, 0.f, 0.f, 0.f);
    float2 t01 = make_float2(0.f, 0.f), t23 = make_float2(0.f, 0.f);
    if (has_t) {
        const uint2 raw = reinterpret_cast<const uint2 *>(o_t + size_t(unit) * 128)[lane];
        t01 = __half22float2(*reinterpret_cast<const __half2 *>(&raw.x));
        t23 = __half22float2(*reinterpret_cast<const __half2 *>(&raw.y));
    }
    const __half2 r01 = __floats2half2_rn((wp * a.x + wt * t01.x) * inv, (wp * a.y + wt * t01.y) * inv);
    const __half2 r23 = __floats2half2_rn((wp * a.z + wt * t23.x) * inv, (wp * a.w + wt * t23.y) * inv);
    uint2 res;
    res.x = *reinterpret_cast<const uint32_t *>(&r01);
    res.y = *reinterpret_cast<const uint32_t *>(&r23);
    reinterpret_cast<uint2 *>(out + size_t(unit) * 128)[lane] = res;
}

// Workspace of pa_decode_grouped: the decode's own split-K workspace, then
// the prefix part's fp32 outputs and lse, the tail part's outputs and lse,
// the tail tables, tail lengths and each member's prefix length.
struct GroupedLayout {
    size_t dec, o_p, lse_p, o_t, lse_t, tables, tlens, pref, total;
};

GroupedLayout grouped_layout(int num_seqs, int num_heads, int head_dim, int max_blocks)
{
    GroupedLayout w{};
    const size_t units = size_t(num_seqs) * size_t(num_heads);
    w.dec = 0;
    w.o_p = align256(pa_decode_workspace_size(num_seqs, num_heads, head_dim, 0));
    w.lse_p = w.o_p + align256(units * head_dim * sizeof(float));
    w.o_t = w.lse_p + align256(units * sizeof(float));
    w.lse_t = w.o_t + align256(units * head_dim * 2);
    w.tables = w.lse_t + align256(units * sizeof(float));
    w.tlens = w.tables + align256(size_t(num_seqs) * size_t(max_blocks) * sizeof(int32_t));
    w.pref = w.tlens + align256(size_t(num_seqs) * sizeof(int32_t));
    w.total = w.pref + align256(size_t(num_seqs) * sizeof(int32_t));
    return w;
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
                          num_heads, head_dim, block_size, num_blocks, scale, false, nullptr,
                          nullptr, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" size_t pa_decode_grouped_workspace_size(int num_seqs, int num_heads, int head_dim,
                                                   int max_blocks_per_seq)
{
    if (num_seqs < 0 || num_heads < 0 || head_dim < 0 || max_blocks_per_seq < 0)
        return 0;
    return grouped_layout(num_seqs, num_heads, head_dim, max_blocks_per_seq).total;
}

extern "C" pa_status pa_decode_grouped(void *out, const void *q, const void *k_cache,
                                       const void *v_cache, const int32_t *block_tables,
                                       int max_blocks_per_seq, const int32_t *context_lens,
                                       int max_context_len, const int32_t *group_start,
                                       const int32_t *prefix_lens, int num_groups,
                                       int max_group_size, int num_seqs, int num_heads,
                                       int head_dim, int block_size, int num_blocks, float scale,
                                       void *workspace, size_t workspace_bytes, pa_stream_t stream)
{
    if (num_seqs < 0 || num_groups < 0 || max_group_size < 0 || num_heads <= 0 ||
        num_blocks <= 0 || max_context_len < 0 || max_blocks_per_seq < 0)
        return PA_ERR_INVALID_ARG;
    if (head_dim != pa::kPD || !supported_block_size(block_size))
        return PA_ERR_UNSUPPORTED;
    if (int64_t(max_context_len) > int64_t(max_blocks_per_seq) * block_size ||
        !std::isfinite(scale) || !(scale > 0.f) || (num_seqs > 0 && num_groups == 0) ||
        num_groups > num_seqs)
        return PA_ERR_INVALID_ARG;
    if (num_seqs == 0)
        return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !group_start ||
        !prefix_lens || max_group_size == 0)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
        (reinterpret_cast<uintptr_t>(context_lens) & 3u) ||
        (reinterpret_cast<uintptr_t>(group_start) & 3u) ||
        (reinterpret_cast<uintptr_t>(prefix_lens) & 3u))
        return PA_ERR_INVALID_ARG;
    if (num_seqs > 65535 || num_heads > 65535 ||
        int64_t(num_blocks) * num_heads * block_size > INT32_MAX)
        return PA_ERR_INVALID_ARG;
    const GroupedLayout w = grouped_layout(num_seqs, num_heads, head_dim, max_blocks_per_seq);
    if (!workspace || workspace_bytes < w.total || !aligned16(workspace))
        return PA_ERR_WORKSPACE;
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    float *o_p = reinterpret_cast<float *>(ws + w.o_p);
    float *lse_p = reinterpret_cast<float *>(ws + w.lse_p);
    __half *o_t = reinterpret_cast<__half *>(ws + w.o_t);
    float *lse_t = reinterpret_cast<float *>(ws + w.lse_t);
    int32_t *tail_tables = reinterpret_cast<int32_t *>(ws + w.tables);
    int32_t *tail_lens = reinterpret_cast<int32_t *>(ws + w.tlens);
    int32_t *prefix_of = reinterpret_cast<int32_t *>(ws + w.pref);
    unsigned int *err = device_error_word();
    if (!err)
        return PA_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

    // 1. each member's tail table and length
    if (max_group_size > 65535)
        return PA_ERR_INVALID_ARG;
    if (launch_pdl(grouped_tails_kernel, dim3(unsigned(num_groups), unsigned(max_group_size)),
                   dim3(128), 0, s, block_tables,
                   max_blocks_per_seq, context_lens, max_context_len, group_start, prefix_lens,
                   block_size, num_seqs, tail_tables, tail_lens, prefix_of, err) != cudaSuccess)
        return PA_ERR_CUDA;
    // 2. the shared prefix, once per (group, head), on the tensor cores
    pa_status st = launch_prefill(o_t, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                                  prefix_lens, max_context_len, group_start, num_seqs,
                                  max_group_size, num_groups, num_heads, head_dim, block_size,
                                  num_blocks, scale, true, o_p, lse_p, s);
    if (st != PA_OK)
        return st;
    // 3. each member's own tail
    st = pa_host::decode_with_lse(o_t, q, k_cache, v_cache, tail_tables, max_blocks_per_seq, tail_lens,
                         max_context_len, num_seqs, num_heads, head_dim, block_size, num_blocks,
                         scale, ws + w.dec, w.o_p - w.dec, lse_t, stream);
    if (st != PA_OK)
        return st;
    // 4. merge the two parts
    const int units = num_seqs * num_heads;
    return launch_pdl(grouped_merge_kernel, dim3(unsigned((units + 7) / 8)), dim3(256), 0, s,
                      static_cast<__half *>(out), static_cast<const float *>(o_p),
                      static_cast<const float *>(lse_p), static_cast<const __half *>(o_t),
                      static_cast<const float *>(lse_t), static_cast<const int32_t *>(prefix_of),
                      static_cast<const int32_t *>(tail_lens), num_heads, units) == cudaSuccess
               ? PA_OK
               : PA_ERR_CUDA;
}
