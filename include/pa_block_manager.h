/*
 * pa_block_manager.h — host-side KV block manager of libpa (C ABI).
 *
 * The bookkeeping the pages describe around the paged cache:
 *   - polomodov.tech "vLLM and PagedAttention", slide 12: one shared pool of
 *     physical blocks instead of per-request reservations; a free block goes
 *     to whoever needs it next.
 *   - slide 11: a new physical block is taken only when the sequence's last
 *     block is full; otherwise the next token goes into the free slot.
 *   - slide 10: the block table maps logical blocks to physical ones.
 *   - comfyai.app "6.4 PagedAttention", 6.4.2-6.4.3 and slide 13: sequences
 *     forked for parallel sampling share their blocks with reference counts;
 *     the first write into a shared block copies it (copy-on-write): the
 *     writer gets a new block (reference count 1), the old block's count drops
 *     by one, and only that last block is copied.
 *   - slide 15: preemption is all-or-nothing (the newest request is evicted)
 *     and a preempted request comes back by swapping its blocks out to host
 *     memory and in again, or by recomputation.  The manager keeps a second
 *     pool for swapped blocks and moves whole sequence groups between the
 *     pools; the data itself moves with pa_swap_blocks.
 *
 * Policy choices the pages leave open (fixed here, deterministic):
 *   - free blocks form a stack; a fresh manager hands out 0, 1, 2, ... and a
 *     freed block is the next one handed out;
 *   - sequence ids are caller-chosen 64-bit integers;
 *   - a swap moves a group of sequences that holds every reference to its
 *     blocks (e.g. a request and all its forked samples); each distinct block
 *     gets one block of the other pool, in order of first appearance
 *     (sequences in the given order, each table front to back), keeping its
 *     reference count; the released blocks go back to their pool's stack in
 *     that same order.
 *
 * Ownership: the manager is host memory owned by the caller (create/destroy).
 * Every pointer argument is a HOST pointer.  A manager is safe to use from
 * several threads (calls are serialised internally).  Failing calls change
 * nothing (all-or-nothing).
 */
#ifndef PA_BLOCK_MANAGER_H
#define PA_BLOCK_MANAGER_H

#include <stddef.h>
#include <stdint.h>

#include "pa.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pa_block_manager pa_block_manager;

/* New manager over a pool of num_blocks blocks of block_size tokens.
 * Returns NULL on invalid sizes or host allocation failure. */
PA_API pa_block_manager *pa_bm_create(int num_blocks, int block_size);
/* Same, with a host (swap) pool of num_cpu_blocks blocks (>= 0). */
PA_API pa_block_manager *pa_bm_create_with_swap(int num_blocks, int num_cpu_blocks,
                                                int block_size);
PA_API void pa_bm_destroy(pa_block_manager *bm);

/* Blocks currently in the free pool. */
PA_API int pa_bm_num_free(const pa_block_manager *bm);
/* Reference count of a physical block (0 = free); -1 for an invalid id. */
PA_API int pa_bm_refcount(const pa_block_manager *bm, int block);

/* Blocks free in the host (swap) pool; reference count of a host block
 * (-1 for an invalid id). */
PA_API int pa_bm_num_free_cpu(const pa_block_manager *bm);
PA_API int pa_bm_cpu_refcount(const pa_block_manager *bm, int block);
/* 1 if the sequence's blocks are in the host pool, 0 if on the device, -1 if
 * unknown. */
PA_API int pa_bm_is_swapped(const pa_block_manager *bm, int64_t seq);

/*
 * Swap-out: move the n sequences `seqs` (all on the device) to the host pool.
 * pairs ([max_pairs, 2] int64) receives one (device block, host block) pair
 * per distinct block, for pa_swap_blocks from the device pool to the host
 * pool; *num_pairs is set to the number of distinct blocks even when the call
 * fails for lack of room in `pairs`.  The device blocks return to the free
 * pool.  PA_ERR_INVALID_ARG (nothing changed) for an unknown, repeated or
 * already swapped sequence, a block also held by a sequence outside the
 * group, or max_pairs < *num_pairs; PA_ERR_OUT_OF_BLOCKS if the host pool is
 * short.  Swapped sequences cannot fork, append or appear in block tables
 * until they are swapped in; they can be freed.
 *
 * Swap-in: the reverse, (host block, device block) pairs for pa_swap_blocks
 * from the host pool to the device pool; PA_ERR_OUT_OF_BLOCKS if the device
 * pool is short.
 */
PA_API pa_status pa_bm_swap_out(pa_block_manager *bm, const int64_t *seqs, int n, int64_t *pairs,
                                int max_pairs, int *num_pairs);
PA_API pa_status pa_bm_swap_in(pa_block_manager *bm, const int64_t *seqs, int n, int64_t *pairs,
                               int max_pairs, int *num_pairs);

/* Register sequence `seq` with `prompt_len` tokens already in the cache:
 * takes ceil(prompt_len / block_size) blocks.  PA_ERR_INVALID_ARG if seq
 * exists or prompt_len < 0; PA_ERR_OUT_OF_BLOCKS if the pool is short. */
PA_API pa_status pa_bm_add_sequence(pa_block_manager *bm, int64_t seq, int prompt_len);

/* Parallel sampling: `child` starts as a copy of `parent`'s table and length,
 * sharing every block (each block's reference count + 1).  The parent must be
 * on the device. */
PA_API pa_status pa_bm_fork(pa_block_manager *bm, int64_t parent, int64_t child);

/* Release a sequence: every block's reference count - 1; blocks reaching 0
 * return to the pool. */
PA_API pa_status pa_bm_free_sequence(pa_block_manager *bm, int64_t seq);

/*
 * One decode step for n sequences: reserve the slot of each sequence's next
 * token (position = its current length), then its length grows by one.
 * slots[i] = physical_block * block_size + offset (what pa_reshape_and_cache
 * takes).  When the slot falls into a block shared with other sequences, the
 * block is copied first: the pair (shared, new) is appended to cow_pairs
 * ([n, 2] capacity) for pa_copy_blocks, and *num_pairs is set to their count.
 * All-or-nothing: PA_ERR_OUT_OF_BLOCKS (nothing changed) if the pool cannot
 * cover every new and copied block of the step; PA_ERR_INVALID_ARG for an
 * unknown or repeated sequence id.
 */
PA_API pa_status pa_bm_append_slots(pa_block_manager *bm, const int64_t *seqs, int n,
                                    int64_t *slots, int64_t *cow_pairs, int *num_pairs);

/*
 * Block tables and context lengths for a batch: row i of `block_tables`
 * ([n, max_blocks], int32) gets sequence seqs[i]'s physical block ids, padded
 * with -1; context_lens[i] its length.  PA_ERR_INVALID_ARG if a table does not
 * fit in max_blocks or a sequence is unknown.
 */
PA_API pa_status pa_bm_block_tables(const pa_block_manager *bm, const int64_t *seqs, int n,
                                    int32_t *block_tables, int max_blocks, int32_t *context_lens);

#ifdef __cplusplus
}
#endif

#endif /* PA_BLOCK_MANAGER_H */
