/*
 * pagedkv_block_manager.h - host-side block manager for a paged KV cache
 * (C ABI; plain C++, no CUDA).
 *
 * What it keeps, after the pages: a pool of fixed-size physical blocks with
 * a free list and a reference count per block ("啃透vLLM源码", §2.2,
 * PhysicalTokenBlock's ref_count "for sharing"); a block table per sequence
 * mapping logical block i to a physical id, blocks taken from the free list
 * when a sequence needs one and returned when it finishes ("vLLM基础", §2.3);
 * the scheduler's admission test, "can the pool give this many blocks"
 * ("啃透vLLM源码", §3, schedule / can_allocate); in-order filling of a
 * sequence's last block ("啃透vLLM源码", §2.2, append_tokens); and
 * copy-on-write: sequences forked from one another share physical blocks
 * until one of them writes into a shared block, which is then copied
 * ("vLLM基础", §2.3).
 *
 * It produces exactly the integer inputs of a decode step: block tables,
 * context lengths, the slot of each new token (pa_write_kv) and the
 * (src, dst) block pairs to duplicate first (pa_copy_blocks).
 *
 * Conventions: ids of sequences are caller-chosen int64 keys. Every call
 * returns a pa_status (PA_ERR_INVALID_ARG for an unknown or duplicate
 * sequence, a bad argument or an exhausted pool; pa_last_error() says which)
 * and leaves the manager unchanged when it fails. A manager is not safe to
 * use from two threads at once; distinct managers are independent.
 */
#ifndef PAGEDKV_BLOCK_MANAGER_H
#define PAGEDKV_BLOCK_MANAGER_H

#include <stddef.h>
#include <stdint.h>

#include "pagedkv.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pa_block_manager pa_block_manager;

/* A pool of num_blocks blocks of block_size tokens. free_order (may be NULL)
 * is a permutation of 0..num_blocks-1 giving the order in which free blocks
 * are handed out; NULL means ascending ids. Returns NULL on bad arguments or
 * allocation failure. */
pa_block_manager *pa_bm_create(int32_t num_blocks, int32_t block_size,
                               const int32_t *free_order);
void pa_bm_destroy(pa_block_manager *bm);

int32_t pa_bm_num_free(const pa_block_manager *bm);
/* 1 if n more blocks can be handed out now, else 0 (admission control). */
int32_t pa_bm_can_allocate(const pa_block_manager *bm, int32_t n);
/* The reference count of a block (0 = free), -1 for an id outside the pool. */
int32_t pa_bm_ref_count(const pa_block_manager *bm, int32_t block);

/* A new, empty sequence. */
pa_status pa_bm_add_sequence(pa_block_manager *bm, int64_t seq);
/* Reserve room for n more tokens of seq (a prompt, a suffix): fills the
 * last block first, then takes fresh blocks. Fails without change if the
 * last block is shared or the pool cannot give the blocks needed. */
pa_status pa_bm_allocate_tokens(pa_block_manager *bm, int64_t seq, int32_t n);
/* A new sequence `child` holding the same blocks and tokens as `parent`
 * (every block's reference count goes up by one). */
pa_status pa_bm_fork(pa_block_manager *bm, int64_t parent, int64_t child);
/* Append one token: a fresh block when the last one is full; a copy of the
 * last block first when it is shared (copy-on-write). *slot receives
 * block * block_size + offset; *cow_src / *cow_dst the copied pair, or -1. */
pa_status pa_bm_append_token(pa_block_manager *bm, int64_t seq, int64_t *slot,
                             int64_t *cow_src, int64_t *cow_dst);
/* Return every block of seq and forget it. */
pa_status pa_bm_free_sequence(pa_block_manager *bm, int64_t seq);

/* Tokens held by seq, or -1 if unknown. */
int32_t pa_bm_num_tokens(const pa_block_manager *bm, int64_t seq);
/* Copy seq's block table into out[0..cap); returns its length (which may
 * exceed cap), or -1 if seq is unknown. */
int32_t pa_bm_block_table(const pa_block_manager *bm, int64_t seq, int32_t *out, int32_t cap);

/* One decode step for n sequences: append one token to each (in the order
 * given) and fill the step's inputs.
 *   block_tables   host int32 [n][max_blocks_per_seq], -1 past each table
 *   context_lens   host int32 [n], tokens after the append
 *   slot_mapping   host int64 [n], slot of each new token
 *   copy_pairs     host int64 [n][2], (src, dst) to copy before writing;
 *                  *num_pairs receives how many were filled
 * Checks first that the pool can give every block the step needs and that
 * every table fits max_blocks_per_seq; fails without change otherwise. */
pa_status pa_bm_prepare_decode(pa_block_manager *bm, const int64_t *seqs, int32_t n,
                               int32_t max_blocks_per_seq, int32_t *block_tables,
                               int32_t *context_lens, int64_t *slot_mapping,
                               int64_t *copy_pairs, int32_t *num_pairs);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_BLOCK_MANAGER_H */
