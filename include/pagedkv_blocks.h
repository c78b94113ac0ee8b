/*
 * pagedkv_blocks.h -- C ABI of the host-side block manager in libpagedkv.so:
 * it hands out the physical blocks of a paged KV pool to sequences, shares
 * full blocks between sequences with the same token prefix, and produces the
 * block tables, context lengths and slot mappings that pkv_store_kvcache and
 * pkv_paged_attention_decode consume.
 *
 * The operation, from the pages: the block manager divides the KV memory
 * into fixed-size blocks, gives each request the blocks it needs and takes
 * them back when the request ends so that others can reuse them
 * ("Nano-vLLM：轻量高效的大模型推理框架", section 三.1, 块管理器); when
 * requests share a prefix, the prefix's cached KV is reused instead of being
 * recomputed -- each request's prefix is hashed, a hit reuses the cached
 * blocks, a miss computes and caches them (same page, section 三.2 (1)
 * 前缀缓存); block tables map logical to physical blocks and KV blocks are
 * shared within and across requests ("DeepSeek复刻vLLM反超原版", section
 * "vLLM：大模型推理的加速引擎与挑战").
 *
 * Policy (readings where the pages are silent):
 *  - Only full blocks are shared, and matching stops at the first block that
 *    misses. Block i of a sequence is identified by its tokens and by
 *    everything before it: a 128-bit chain key over the prefix, with the
 *    block's own tokens and its parent's key compared on a hit, so two
 *    sequences share block i when their first (i + 1) * block_size tokens
 *    are equal (and otherwise only if two different prefixes collide in all
 *    128 bits of their parents' keys). Registering a prefix that is already
 *    cached moves its entry to the newer block.
 *  - Free blocks form a queue: initially 0, 1, ..., num_blocks - 1; a block
 *    whose last user leaves goes to the back; a new block is taken from the
 *    front. A freed full block keeps its cache entry until it is taken again,
 *    so a later request with the same prefix can still hit it (a hit on a
 *    free block takes it out of the queue).
 *  - A partial last block is private to its sequence; when appending a token
 *    fills it, it becomes a cached full block that later sequences can share.
 *  - A sequence's blocks are released last block first, so the tail of a
 *    cached prefix is reused before its head.
 *
 * Contract with the caller: a full block is shared from the moment it is
 * registered (when add_sequence takes it for a prompt, or when append_token
 * fills it), while its K/V is written by the caller's store_kvcache. A
 * sequence that hits a block must therefore attend only after the K/V of
 * that block has been stored (stream order does it within one step; with
 * chunked prefill, admit requests that could hit a prompt's blocks after
 * those blocks have been prefilled).
 *
 * Ownership: the manager owns its state; every call is synchronous host code
 * and the manager is not thread-safe (one caller at a time). Errors are
 * returned as pkv_status values (pagedkv.h); a failed call changes nothing.
 */
#ifndef PAGEDKV_BLOCKS_H
#define PAGEDKV_BLOCKS_H

#include <stddef.h>
#include <stdint.h>

#include "pagedkv.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pkv_block_manager pkv_block_manager; /* opaque */

/* New manager over num_blocks blocks of block_size tokens; NULL on bad sizes
 * (either below 1, or num_blocks * block_size slots not fitting in int32). */
PKV_API pkv_block_manager *pkv_bm_create(int64_t num_blocks, int block_size);
PKV_API void pkv_bm_destroy(pkv_block_manager *bm);

/*
 * Add sequence seq_id (any id not in use) with its prompt tokens: leading full
 * blocks whose prefix is cached are shared, the rest get new blocks.
 * *num_cached_tokens receives how many leading tokens already have their KV
 * in the pool (a multiple of block_size, possibly all of them; their KV need
 * not be written again).
 * PKV_ERR_INVALID_ARG: id in use, num_tokens < 1, null pointers.
 * PKV_ERR_WORKSPACE: not enough free blocks (nothing is allocated).
 */
PKV_API int pkv_bm_add_sequence(pkv_block_manager *bm, int64_t seq_id, const int32_t *tokens,
                                int num_tokens, int *num_cached_tokens);

/*
 * Append one token to seq_id (its KV is about to be written): a new block is
 * taken when the last one is full. *slot receives the token's slot
 * (block * block_size + offset) for pkv_store_kvcache.
 * PKV_ERR_WORKSPACE when a block is needed and none is free.
 */
PKV_API int pkv_bm_append_token(pkv_block_manager *bm, int64_t seq_id, int32_t token, int64_t *slot);

/* Remove seq_id; its blocks go back to the free queue when no one else uses them. */
PKV_API int pkv_bm_free_sequence(pkv_block_manager *bm, int64_t seq_id);

/*
 * Block table row of seq_id: blocks in logical order, padded with -1 up to
 * max_blocks (PKV_ERR_INVALID_ARG if it does not fit); *num_tokens receives
 * the sequence's length (its context length), also when the row does not
 * fit, so max_blocks = 0 asks for the length alone.
 */
PKV_API int pkv_bm_block_table(const pkv_block_manager *bm, int64_t seq_id, int32_t *row, int max_blocks,
                               int *num_tokens);

/* Slots of positions [start, start + count) of seq_id (for pkv_store_kvcache);
 * PKV_ERR_INVALID_ARG unless 0 <= start <= start + count <= its length. */
PKV_API int pkv_bm_slots(const pkv_block_manager *bm, int64_t seq_id, int start, int count, int32_t *slots);

/* Number of free blocks (including freed blocks still holding a cached prefix). */
PKV_API int64_t pkv_bm_num_free_blocks(const pkv_block_manager *bm);

/* How many live sequences use physical block `block` (0 when free). */
PKV_API int pkv_bm_block_refcount(const pkv_block_manager *bm, int64_t block, int *refcount);

/*
 * One decode step's bookkeeping in one call (host arrays of n entries):
 * append tokens[i] to sequence seq_ids[i] and write its slot to slots[i]
 * (the slot_mapping of pkv_store_kvcache). The ids must be distinct and
 * live. All or nothing: PKV_ERR_INVALID_ARG (unknown or repeated id) or
 * PKV_ERR_WORKSPACE (fewer free blocks than the step needs) leave every
 * sequence as it was.
 */
PKV_API int pkv_bm_append_tokens(pkv_block_manager *bm, const int64_t *seq_ids, const int32_t *tokens, int n,
                                 int32_t *slots);

/*
 * The decode inputs of n sequences: block_tables is [n][max_blocks] int32
 * (row i = seq_ids[i]'s blocks, padded with -1) and context_lens[i] its
 * length. PKV_ERR_INVALID_ARG for an unknown id or a row longer than
 * max_blocks (the outputs are then partly written; the manager is unchanged).
 */
PKV_API int pkv_bm_block_tables(const pkv_block_manager *bm, const int64_t *seq_ids, int n, int32_t *block_tables,
                                int max_blocks, int32_t *context_lens);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_BLOCKS_H */
