/*
 * Host block manager for the paged KV cache: the bookkeeping that produces the
 * block tables, context lengths and slot mappings the kernels of
 * pagedattn.h consume, and the block copies that copy-on-write needs.
 *
 * Passages: nano-vllm (ovshake) README, "Key Concepts Explained:
 * PagedAttention" (blocks of one pool, allocated on demand, a per-sequence
 * list of blocks), "Features" ("Block-based Memory Management: zero memory
 * waste with on-demand allocation", "Prefix Caching: share KV cache blocks
 * for common prefixes", "Preemption"), and the project layout's
 * core/block.py and core/block_manager.py.  The pages give no interface; the
 * one below is this library's.
 *
 * Model.  A pool of num_blocks physical blocks of block_size token slots.
 * A sequence (identified by a caller-chosen int64 id) owns a list of blocks
 * holding its positions 0 .. len-1 in order: position t is slot
 * blocks[t / block_size] * block_size + t % block_size.  Blocks carry a
 * reference count: the number of sequences whose list holds them.  A block
 * with count 0 is free.
 *   - Prefix caching: a FULL block whose token ids are known is registered
 *     under a hash of (the previous block's hash, its block_size token ids);
 *     a later sequence whose prompt starts with the same full blocks reuses
 *     them (count + 1) instead of allocating.  Lookups compare the stored
 *     token ids, so a hash collision never shares a wrong block.  A cached
 *     block whose count drops to 0 stays registered (and reusable) until the
 *     allocator hands it out again; free blocks are handed out in the order
 *     they were freed (never-used blocks first, in id order).
 *   - fork: a child sequence shares all of its parent's blocks.
 *   - Copy-on-write: appending to a sequence whose last block is partly
 *     filled and shared (count > 1) first moves the sequence to a fresh block;
 *     the caller must copy the old block's rows into the new one on the GPU
 *     (pa_copy_blocks, with the (src, dst) pairs returned) before the append
 *     writes the new row.
 *
 * Ownership and errors.  pa_bm_create returns an owned handle (NULL when
 * out of memory or on bad sizes); pa_bm_destroy frees it.  All other calls
 * take the handle and caller-owned host arrays.  Calls on one handle must not
 * run concurrently.  Every call checks all of its arguments, and the
 * capacity, before changing anything: a call that returns an error leaves the
 * manager as it was.  Status codes are pa_status_t values (pagedattn.h):
 * PA_ERR_INVALID for bad handles, unknown or duplicate sequence ids and bad
 * sizes; PA_ERR_WORKSPACE when the pool has too few free blocks (the
 * "out of blocks" condition a scheduler answers with preemption).
 */
#ifndef PAGED_KV_BLOCK_MANAGER_H_
#define PAGED_KV_BLOCK_MANAGER_H_

#include <stddef.h>
#include <stdint.h>

#include "pagedattn.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pa_block_manager pa_block_manager;

pa_block_manager* pa_bm_create(int32_t num_blocks, int32_t block_size);
void pa_bm_destroy(pa_block_manager* bm);

/* Free blocks (count 0), and blocks a new sequence of n tokens would take
 * (the full blocks found in the prefix cache are not counted when token_ids
 * is given). */
int32_t pa_bm_num_free(const pa_block_manager* bm);
int32_t pa_bm_blocks_needed(const pa_block_manager* bm, const int64_t* token_ids, int32_t num_tokens);

/*
 * Register sequence seq_id holding num_tokens positions (a prompt).
 * token_ids (may be NULL): the prompt's token ids; full blocks are looked up
 * in and added to the prefix cache.  *cached_tokens (may be NULL) receives
 * how many leading positions came from the cache (a multiple of block_size):
 * their K/V rows are already in the pool and need not be computed again.
 */
pa_status_t pa_bm_add_sequence(pa_block_manager* bm, int64_t seq_id, const int64_t* token_ids,
                               int32_t num_tokens, int32_t* cached_tokens);

/*
 * One decode step for n sequences: each gets one more position (its length
 * grows by 1) and slots_out[i] receives that position's slot.  token_ids
 * (may be NULL) are the appended tokens; a block they fill is added to the
 * prefix cache.  Copy-on-write pairs go to cow_out[2*k] (src), cow_out[2*k+1]
 * (dst), k < *num_cow (cow_out has room for 2*n entries).  The ids must be
 * distinct.
 */
pa_status_t pa_bm_append_slots(pa_block_manager* bm, const int64_t* seq_ids, const int64_t* token_ids, int32_t n,
                               int64_t* slots_out, int32_t* cow_out, int32_t* num_cow);

/* Child shares every block of parent (same length). */
pa_status_t pa_bm_fork(pa_block_manager* bm, int64_t parent_id, int64_t child_id);

/* Drop the sequence; its blocks' counts go down by one. */
pa_status_t pa_bm_free_sequence(pa_block_manager* bm, int64_t seq_id);

/* Length (positions) of a sequence, or -1 when unknown. */
int32_t pa_bm_length(const pa_block_manager* bm, int64_t seq_id);

/*
 * Block tables and context lengths of n sequences, in the layout the decode
 * calls take: tables_out [n][max_blocks] int32 (-1 past each sequence's last
 * block), lens_out [n] int32.  PA_ERR_INVALID when a sequence holds more
 * than max_blocks blocks.
 */
pa_status_t pa_bm_block_tables(const pa_block_manager* bm, const int64_t* seq_ids, int32_t n, int32_t max_blocks,
                               int32_t* tables_out, int32_t* lens_out);

/* Slots of positions [start, start + count) of a sequence (a prefill's slot
 * mapping); the positions must exist. */
pa_status_t pa_bm_slots(const pa_block_manager* bm, int64_t seq_id, int32_t start, int32_t count,
                        int64_t* slots_out);

/* Reference count of a physical block (-1 for a bad id). */
int32_t pa_bm_ref_count(const pa_block_manager* bm, int32_t block);

/*
 * pa_copy_blocks -- copy whole blocks inside the pool, both caches:
 * k_cache[dst] = k_cache[src], v_cache[dst] = v_cache[src] for each pair
 * (pairs: device int32 [n][2] = (src, dst)), every kv head, row and
 * element: num_kv_heads * block_size * head_dim elements of dtype per block
 * and cache, byte for byte.  Pairs must not overlap (no block is both a
 * source and a destination).  Ids outside [0, num_blocks) raise
 * PA_DEVERR_BLOCK and are skipped.  One launch; asynchronous on stream.
 */
pa_status_t pa_copy_blocks(void* k_cache, void* v_cache, const int32_t* pairs, int32_t n, int32_t num_blocks,
                           int32_t block_size, int32_t num_kv_heads, int32_t head_dim, pa_dtype_t dtype,
                           pa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PAGED_KV_BLOCK_MANAGER_H_ */
