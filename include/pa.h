/*
 * pa.h — C ABI of libpa, the B200 (sm_100a) PagedAttention decode path.
 *
 * The operations follow the pages on PagedAttention:
 *   - comfyai.app "6.4 PagedAttention", 6.4.1 Mechanism: each sequence's
 *     K/V cache is split into blocks of a fixed number of tokens; a block
 *     table maps the sequence's logically contiguous blocks onto physically
 *     non-contiguous blocks of one pool.
 *   - polomodov.tech "vLLM and PagedAttention", slide 9 (the attention kernel
 *     fetches K and V from non-contiguous blocks by their addresses), slide 10
 *     (block table, logical -> physical), slide 11 (a new token goes into the
 *     next free slot; a new block is taken only when the last one is full),
 *     slide 13 (copy-on-write duplicates only the last block).
 *   - brentwoodlivery.com "5.3.18 LLM serving, vLLM, quantized inference":
 *     paging changes only the memory layout, not the attention arithmetic.
 *
 * Layouts (row-major, fp16 = IEEE binary16):
 *   q, out            [num_seqs, num_heads, head_dim]           fp16
 *   key, value        [num_tokens, num_heads, head_dim]         fp16
 *   k_cache, v_cache  [num_blocks, num_heads, block_size, head_dim] fp16
 *                     element (p, h, j, d) at ((p*H + h)*bs + j)*D + d
 *   block_tables      [num_seqs, max_blocks_per_seq]            int32
 *   context_lens      [num_seqs]                                int32
 *   slot_mapping      [num_tokens]   int64, slot = block*bs + offset, <0 = skip
 *   block_mapping     [num_pairs, 2] int64, (src, dst) physical block ids
 *
 * Ownership and execution: every array argument is a DEVICE pointer owned by
 * the caller, and must stay valid until the work on `stream` has finished.
 * The library never allocates device memory.  Calls only validate arguments
 * on the host and enqueue kernels on `stream` (asynchronous); PA_OK means the
 * launch was accepted.  fp16 arrays and the workspace must be 16-byte aligned.
 *
 * Errors: host-detectable problems return a status and launch nothing.
 * Out-of-range indices found on the device (block id >= num_blocks, slot past
 * the pool, context_lens[b] outside [0, max_context_len], a bad copy pair) are
 * never dereferenced: the access is skipped, the affected result is
 * unspecified, and a bit is set in a per-device error word read (and
 * cleared) by pa_get_last_device_error().
 */
#ifndef PA_H
#define PA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as the CUDA runtime's cudaStream_t; NULL = legacy default stream. */
typedef struct CUstream_st *pa_stream_t;

typedef enum pa_status {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1,  /* null pointer, negative size, misalignment, lengths too long */
    PA_ERR_UNSUPPORTED = 2,  /* head_dim not in {64,128} or block_size not in {8,16,32,64,128} */
    PA_ERR_CUDA = 3,         /* the CUDA runtime refused the launch */
    PA_ERR_WORKSPACE = 4,    /* workspace null or smaller than pa_decode_workspace_size() */
    PA_ERR_OUT_OF_BLOCKS = 5 /* block manager: the free pool cannot cover the request */
} pa_status;

/* Bits of the device error word (pa_get_last_device_error). */
#define PA_DEVERR_BLOCK_ID    1u   /* decode: block table entry outside [0, num_blocks) */
#define PA_DEVERR_CONTEXT_LEN 2u   /* decode: context_lens[b] < 0 or > max_context_len */
#define PA_DEVERR_SLOT        4u   /* cache write: slot >= num_blocks * block_size (decode_append: or not the slot of position L - 1) */
#define PA_DEVERR_COPY_PAIR   8u   /* copy: src or dst outside [0, num_blocks) */
#define PA_DEVERR_TIMEOUT     16u  /* decode: a shared-memory transfer did not arrive in ~1 s */

/*
 * Cache write (polomodov.tech slide 11; comfyai.app 6.4.1).  For every token i
 * with slot = slot_mapping[i] >= 0, copy key[i, h, :] to
 * k_cache[slot / block_size, h, slot % block_size, :] and value[i, h, :] to
 * v_cache at the same place, for all heads h.  Negative slots (padding) are
 * skipped.  Bit-exact copy.  Slots within one call must be distinct (else
 * which token lands is unspecified).  num_tokens == 0 is a no-op.
 */
PA_API pa_status pa_reshape_and_cache(const void *key, const void *value, void *k_cache,
                               void *v_cache, const int64_t *slot_mapping,
                               int num_tokens, int num_heads, int head_dim,
                               int block_size, int num_blocks, pa_stream_t stream);

/*
 * Bytes of workspace pa_decode needs for these sizes: partial results of the
 * (sequence, head) pairs whose context is split between workers (a fixed
 * part, 2 * 4096 * (head_dim + 2) floats) and one merge ticket per
 * (sequence, head).  Never 0; max_context_len does not change it.
 */
PA_API size_t pa_decode_workspace_size(int num_seqs, int num_heads, int head_dim,
                                int max_context_len);

/*
 * Zero the workspace's merge counters (a cudaMemsetAsync on `stream`).  Call
 * once on a fresh workspace before its first pa_decode, and again after
 * pa_get_last_device_error reported PA_DEVERR_TIMEOUT.  pa_decode leaves the
 * counters at zero when it completes, so a workspace is reusable across calls
 * of any size that fits it.
 */
PA_API pa_status pa_decode_workspace_init(void *workspace, size_t workspace_bytes,
                                   pa_stream_t stream);

/*
 * Paged single-token decode attention (comfyai.app 6.4.1; polomodov.tech
 * slides 9-10; brentwoodlivery.com 5.3.18).  For every sequence b and head h,
 * with L = context_lens[b] and, for t < L,
 *     K_t = k_cache[block_tables[b][t / bs], h, t % bs, :]   (V_t likewise)
 *     s_t = scale * sum_d q[b,h,d] * K_t[d]
 *     out[b,h,:] = sum_t exp(s_t - max s) V_t / sum_t exp(s_t - max s)
 * computed with fp32 accumulation and written as fp16 (round to nearest even).
 * L == 0 writes zeros.  Only block_tables[b][0 .. ceil(L/bs)) is read; cache
 * rows at positions >= L are never used.  max_context_len is a host-side
 * upper bound of context_lens (it sizes the grid); it must not exceed
 * max_blocks_per_seq * block_size.  `workspace` (workspace_bytes >=
 * pa_decode_workspace_size(...), counters zeroed by pa_decode_workspace_init)
 * holds split-K partials; calls that share a workspace must not overlap on
 * the GPU.  Results are deterministic (fixed reduction order, no float
 * atomics), so aliased and copied blocks give bit-identical outputs.
 */
PA_API pa_status pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *block_tables, int max_blocks_per_seq,
                    const int32_t *context_lens, int max_context_len, int num_seqs,
                    int num_heads, int head_dim, int block_size, int num_blocks,
                    float scale, void *workspace, size_t workspace_bytes,
                    pa_stream_t stream);

/*
 * pa_reshape_and_cache of each sequence's newest token followed by pa_decode,
 * in ONE launch (the cache write of a decode step, polomodov.tech "vLLM and
 * PagedAttention" slide 11, fused into the attention that reads it).  For a
 * sequence b with slot_mapping[b] >= 0, position context_lens[b] - 1 is its
 * new token: key[b] / value[b] ([num_seqs, H, D] fp16, device) are written
 * to the cache at slot_mapping[b], which must be the slot the block table
 * gives that position (else PA_DEVERR_SLOT; a slot outside the pool is not
 * written), and the attention uses them for that position.  slot_mapping[b]
 * < 0: no new token, plain decode of the cached context.  Outputs and cache
 * contents are those of the two separate calls.  fp16 caches only; other
 * arguments, layouts and errors as pa_decode.
 */
PA_API pa_status pa_decode_append(void *out, const void *q, const void *key, const void *value,
                                  void *k_cache, void *v_cache, const int64_t *slot_mapping,
                                  const int32_t *block_tables, int max_blocks_per_seq,
                                  const int32_t *context_lens, int max_context_len, int num_seqs,
                                  int num_heads, int head_dim, int block_size, int num_blocks,
                                  float scale, void *workspace, size_t workspace_bytes,
                                  pa_stream_t stream);

/*
 * Copy-on-write block copy (comfyai.app 6.4.2-6.4.3; polomodov.tech slide
 * 13).  For each pair (src, dst): k_cache[dst] = k_cache[src] and
 * v_cache[dst] = v_cache[src], all num_heads * block_size * head_dim
 * elements, bit-exact.  dst ids must be distinct and no dst may also be a
 * src in the same call.  num_pairs == 0 is a no-op.
 */
PA_API pa_status pa_copy_blocks(void *k_cache, void *v_cache, const int64_t *block_mapping,
                         int num_pairs, int num_heads, int head_dim, int block_size,
                         int num_blocks, pa_stream_t stream);

/*
 * Contiguous-cache baseline (polomodov.tech "vLLM and PagedAttention", slide
 * 19: the paged kernel against one that reads a contiguous cache).  The same
 * decode as pa_decode, but over K / V kept contiguous per (sequence, head):
 *   k, v  [num_seqs, num_heads, seq_stride, head_dim] fp16, token t of
 *         sequence b, head h at ((b * H + h) * seq_stride + t) * D,
 * so every address follows from the position and no block table is read.
 * It exists to measure what the paged layout's indirection costs; results
 * equal pa_decode's over the same values.  max_context_len <= seq_stride;
 * the workspace is pa_decode's (pa_decode_workspace_size, zeroed once).
 * Other rules as pa_decode.
 */
PA_API pa_status pa_decode_contiguous(void *out, const void *q, const void *k, const void *v,
                                      const int32_t *context_lens, int max_context_len,
                                      int seq_stride, int num_seqs, int num_heads, int head_dim,
                                      float scale, void *workspace, size_t workspace_bytes,
                                      pa_stream_t stream);

/*
 * pa_decode without a caller-supplied workspace, for callers that cannot
 * allocate device memory at decode time (for example a serving engine that
 * has reserved nearly all free HBM for its KV block pool, or a loop that
 * must not let cudaMalloc/cudaFree synchronise the device).  There is no
 * counterpart on the pages: it is a library convenience.  Same arguments and
 * results as pa_decode minus workspace/workspace_bytes.
 *   - Scratch is a static 8 MiB device array inside libpa, present on every
 *     GPU that loads the library until the process exits; no device memory
 *     is allocated by this call.
 *   - Sizes whose pa_decode_workspace_size() exceeds 8 MiB return
 *     PA_ERR_WORKSPACE (use pa_decode with your own workspace instead).
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.  Each call clears the merge counters with a
 *     cudaMemsetAsync on `stream`.
 *   - All calls on a device share the one array: calls that overlap on the
 *     GPU (other streams, other host threads) race and give wrong results.
 *   - The looked-up address is kept per device ordinal for the life of the
 *     process: do not use the library across a cudaDeviceReset (the same
 *     holds for the device error word and the prefill scheduling counters).
 */
PA_API pa_status pa_decode_no_alloc(void *out, const void *q, const void *k_cache,
                                    const void *v_cache, const int32_t *block_tables,
                                    int max_blocks_per_seq, const int32_t *context_lens,
                                    int max_context_len, int num_seqs, int num_heads,
                                    int head_dim, int block_size, int num_blocks, float scale,
                                    pa_stream_t stream);

/*
 * Low-bit KV cache (brentwoodlivery.com "5.3.18 LLM serving, vLLM, quantized
 * inference": the KV cache kept in low-bit integer form with affine
 * quantization s = (r_max - r_min) / (2^b - 1), z = round(-r_min / s),
 * q = round(r / s) + z, r_hat = s (q - z), one (s, z) per group of values).
 * Here b = 8 and a group is one (token, head) row of head_dim values:
 *   k_codes, v_codes    [num_blocks, num_heads, block_size, head_dim] uint8
 *   k_params, v_params  [num_blocks, num_heads, block_size, 2] float (s, z)
 * Rounding decisions are taken in fp32 (IEEE division, round half to even);
 * codes are clamped to [0, 255]; a row whose values are all equal (c) is
 * stored with s = |c| (1 if c = 0) and reconstructs exactly.  Rows holding
 * inf or NaN get unspecified codes.  All arrays are device pointers, 16-byte
 * aligned.
 *
 * pa_reshape_and_cache_int8: quantize each token's key/value rows and store
 * them at their slots (same slot rules as pa_reshape_and_cache).
 */
PA_API pa_status pa_reshape_and_cache_int8(const void *key, const void *value, void *k_codes,
                                           void *v_codes, void *k_params, void *v_params,
                                           const int64_t *slot_mapping, int num_tokens,
                                           int num_heads, int head_dim, int block_size,
                                           int num_blocks, pa_stream_t stream);

/*
 * pa_decode over the int8 cache: K_t and V_t are the dequantized rows
 * s (q - z); otherwise identical to pa_decode (same arguments, workspace,
 * tolerance and determinism).  Moves about half the bytes of pa_decode.
 */
PA_API pa_status pa_decode_int8(void *out, const void *q, const void *k_codes,
                                const void *v_codes, const void *k_params, const void *v_params,
                                const int32_t *block_tables, int max_blocks_per_seq,
                                const int32_t *context_lens, int max_context_len, int num_seqs,
                                int num_heads, int head_dim, int block_size, int num_blocks,
                                float scale, void *workspace, size_t workspace_bytes,
                                pa_stream_t stream);

/*
 * pa_decode_append over the int8 cache (the new token goes into the next
 * free slot: polomodov.tech "vLLM and PagedAttention", slide 11; low-bit
 * KV cache with affine (s, z) per row: brentwoodlivery.com 5.3.18): one
 * launch that quantizes each
 * sequence's new K/V row (key, value [num_seqs, H, D] fp16, exactly as
 * pa_reshape_and_cache_int8 does), writes its codes and (s, z) to
 * slot_mapping[b] (int64, device; negative = nothing to append) and decodes
 * the sequence over its context including that row.  The slot must be the
 * one the block table gives position context_lens[b] - 1, else
 * PA_DEVERR_SLOT is recorded (a slot outside the pool is not written).
 * Outputs and cache contents equal those of pa_reshape_and_cache_int8
 * followed by pa_decode_int8.  Other arguments, layouts, ownership and
 * errors as pa_decode_int8.
 */
PA_API pa_status pa_decode_append_int8(void *out, const void *q, const void *key,
                                       const void *value, void *k_codes, void *v_codes,
                                       void *k_params, void *v_params,
                                       const int64_t *slot_mapping, const int32_t *block_tables,
                                       int max_blocks_per_seq, const int32_t *context_lens,
                                       int max_context_len, int num_seqs, int num_heads,
                                       int head_dim, int block_size, int num_blocks, float scale,
                                       void *workspace, size_t workspace_bytes,
                                       pa_stream_t stream);

/*
 * Copy-on-write copy of whole blocks of any per-block byte size (use it for
 * the int8 codes and their parameter arrays): for each (src, dst) pair, the
 * block_bytes bytes of block src are copied to block dst of `cache`
 * ([num_blocks, block_bytes / elem] contiguous).  block_bytes must be a
 * multiple of 16; same pair rules as pa_copy_blocks.
 */
PA_API pa_status pa_copy_blocks_raw(void *cache, size_t block_bytes, const int64_t *block_mapping,
                                    int num_pairs, int num_blocks, pa_stream_t stream);

/*
 * Swap of whole blocks between two pools, typically the device pool and a
 * pool in page-locked host memory (polomodov.tech "vLLM and PagedAttention",
 * slide 15: a preempted request is brought back by swapping its blocks or by
 * recomputing them).  For each pair i, block block_mapping[2i] of `src`
 * (num_src_blocks blocks of block_bytes bytes) is copied to block
 * block_mapping[2i+1] of `dst` (num_dst_blocks blocks).  Host pools must be
 * device-addressable: allocated with cudaHostAlloc / cudaMallocHost or
 * registered with cudaHostRegister (mapped at the same address, as under
 * unified addressing); a pointer that is neither device memory nor such host
 * memory is refused with PA_ERR_INVALID_ARG.  One call moves one pool array: call it
 * for the K and the V cache (and, for int8 caches, their parameter arrays,
 * with their own block_bytes).  block_mapping [num_pairs, 2] int64 lives in
 * device-addressable memory and the pairs the host block manager's
 * pa_bm_swap_out / pa_bm_swap_in emit fit it directly.  src and dst must be
 * distinct arrays (PA_ERR_INVALID_ARG otherwise), 16-byte aligned, and
 * block_bytes a multiple of 16.  A pair outside the pools is skipped and
 * reported in the device error word (PA_DEVERR_COPY_PAIR).
 */
PA_API pa_status pa_swap_blocks(const void *src, void *dst, size_t block_bytes,
                                const int64_t *block_mapping, int num_pairs, int num_src_blocks,
                                int num_dst_blocks, pa_stream_t stream);

/*
 * Multi-query paged attention: prefill and chunked prefill
 * (brentwoodlivery.com "5.3.18 …": prefill processes all prompt tokens at
 * once and is compute-bound; comfyai.app "6.4 PagedAttention", 6.4.3).
 * Sequence b holds L = context_lens[b] tokens in the cache (already written
 * with pa_reshape_and_cache), the last n_b = query_start_loc[b+1] -
 * query_start_loc[b] of which are new.  New token i of b, at position
 * p = L - n_b + i, attends causally to the cached tokens t <= p:
 *     out[row] = softmax_t(scale q[row].K_t) V_t,  row = query_start_loc[b] + i.
 *   q, out           [num_tokens, num_heads, head_dim] fp16 (device)
 *   query_start_loc  [num_seqs + 1] int32 (device), query_start_loc[0] = 0
 *   max_query_len    host-side bound on n_b (sizes the grid)
 * Runs on the tensor cores (tcgen05, fp16 inputs, fp32 accumulation; the
 * attention weights enter the P.V product rounded to fp16).  head_dim must
 * be 128 (else PA_ERR_UNSUPPORTED); scale must be finite and > 0 (else
 * PA_ERR_INVALID_ARG).  The kernel hands out its work through one of 64
 * per-device counters taken in turn, so at most 64 pa_prefill launches may be
 * in flight on one device at a time (for example on different streams).
 * n_b > L_b is reported in the device
 * error word (PA_DEVERR_CONTEXT_LEN) and that sequence is skipped.
 */
PA_API pa_status pa_prefill(void *out, const void *q, const void *k_cache, const void *v_cache,
                            const int32_t *block_tables, int max_blocks_per_seq,
                            const int32_t *context_lens, int max_context_len,
                            const int32_t *query_start_loc, int num_tokens, int max_query_len,
                            int num_seqs, int num_heads, int head_dim, int block_size,
                            int num_blocks, float scale, pa_stream_t stream);

/*
 * Decode of groups of sequences that share the first blocks of their context
 * -- parallel samples of one prompt, beam candidates (comfyai.app "6.4
 * PagedAttention", 6.4.2; polomodov.tech "vLLM and PagedAttention", slides
 * 13-14: candidates share a prefix of blocks like processes after fork).
 * Same result as pa_decode over the same arguments, but each shared prefix
 * is read from memory once per (group, head): the group's queries are scored
 * against it together on the tensor cores, each member's own tail is scored
 * alone by the decode kernel on the other SMs at the same time, and the
 * parts are merged by their softmax normalisers.
 *   group_start [num_groups + 1] int32 (device): group g = sequences
 *     group_start[g] .. group_start[g+1] - 1; group_start[0] = 0 and
 *     group_start[num_groups] = num_seqs, nondecreasing (every sequence in
 *     exactly one group).
 *   prefix_lens [num_groups] int32 (device): tokens shared by group g, a
 *     multiple of block_size, at most every member's context length; the
 *     members' block tables must agree on those blocks (0 = nothing shared).
 *   max_group_size: host bound on group sizes (<= 65535).
 *   workspace: pa_decode_grouped_workspace_size(num_seqs, num_groups,
 *     num_heads, head_dim, max_context_len, max_blocks_per_seq) bytes,
 *     16-byte aligned, all zero before its first use (cudaMemsetAsync, or
 *     pa_decode_workspace_init); every call leaves it ready for the next,
 *     and one workspace serves any smaller problem too.  Calls that share a
 *     workspace must not overlap on the GPU.
 * head_dim must be 128 (else PA_ERR_UNSUPPORTED), scale > 0.  A prefix that
 * breaks these rules is recorded (PA_DEVERR_CONTEXT_LEN) and its group is
 * decoded without a shared prefix; group bounds outside the batch are
 * recorded and that group is skipped.
 */
PA_API size_t pa_decode_grouped_workspace_size(int num_seqs, int num_groups, int num_heads,
                                               int head_dim, int max_context_len,
                                               int max_blocks_per_seq);
PA_API pa_status pa_decode_grouped(void *out, const void *q, const void *k_cache,
                                   const void *v_cache, const int32_t *block_tables,
                                   int max_blocks_per_seq, const int32_t *context_lens,
                                   int max_context_len, const int32_t *group_start,
                                   const int32_t *prefix_lens, int num_groups, int max_group_size,
                                   int num_seqs, int num_heads, int head_dim, int block_size,
                                   int num_blocks, float scale, void *workspace,
                                   size_t workspace_bytes, pa_stream_t stream);

/* Static description of a status code. */
PA_API const char *pa_status_string(pa_status status);

/*
 * Read and clear the current device's error word (PA_DEVERR_* bits; 0 = no
 * error).  Synchronises with the device.  Returns PA_ERR_CUDA if the read
 * fails, PA_ERR_INVALID_ARG if code is NULL.
 */
PA_API pa_status pa_get_last_device_error(unsigned int *code);

/*
 * Self-test of failure detection (no counterpart on the pages).  Every wait
 * inside the kernels is bounded; this launches one warp that waits on a
 * barrier nothing ever completes, for limit_us microseconds (1 .. 2 000 000),
 * after which it records PA_DEVERR_TIMEOUT in the device error word and
 * exits.  It faults nothing and leaves the context usable.  Asynchronous on
 * `stream`; read the result with pa_get_last_device_error().
 */
PA_API pa_status pa_selftest_bounded_wait(unsigned int limit_us, pa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PA_H */
