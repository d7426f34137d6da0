/*
 * pkv_block_manager.h -- host-side block manager of a paged KV cache (part of libpkv.so).
 *
 * Pages (as in pkv.h):
 *   [KVB] "KV cache, continuous batching and paged attention"
 *   [KVG] "KV cache, GQA, paging and continuous batching"
 *   [INF] inference guide "a2-inf-2"
 *
 * The cache is a pool of num_blocks physical blocks of 16 token slots.  Each sequence owns
 * a block table mapping its logical block j (tokens 16j .. 16j+15) to a physical block;
 * blocks are taken from a free list on demand as the sequence grows and go back when it
 * ends ([KVG] "PagedAttention"; [INF] "PagedAttention: virtual memory for the cache").
 * Only the last block of a sequence can be partly filled ([KVB] "Paged attention").
 *
 * Sharing.  A block may sit in several tables; the manager counts references.
 *   - Forks (parallel samples, beam search) share all of the parent's blocks.  When a
 *     sequence appends into a partly filled block that another table also holds, the
 *     manager first gives it a private copy (copy-on-write at divergence, [KVB] "Paged
 *     attention"; [KVG] "PagedAttention") and reports the (source, copy) pair, which the
 *     caller copies on the GPU with kv_copy_blocks before writing the new tokens.
 *   - Prefix cache ([KVB] "Prefix caching": blocks cached by a hash of the prefix; [INF]
 *     "Prefix caching").  When enabled, every full block whose tokens are known is entered
 *     in a table keyed by (the physical block holding the previous 16 tokens, its
 *     generation, the block's 16 token ids).  The previous block is itself keyed the same
 *     way, so a key identifies the whole prefix up to the block's end exactly: a lookup
 *     never matches a block whose prefix differs, whatever the hash values.  A new
 *     sequence attaches to the longest chain of cached full blocks that matches its
 *     prompt, leaving at least the prompt's last token to be computed (so that prefill
 *     still produces its logits).  Unreferenced cached blocks stay findable until an
 *     allocation needs them; they are then evicted least recently released first.
 *
 * Preemption ([KVG] "The scheduler, and preemption").  pkv_bm_free_blocks gives the number
 * of blocks an allocation can take (free plus evictable), which bounds admission.
 * pkv_bm_swap_out releases a sequence's blocks and reports which ones to copy to host
 * memory with kv_swap_out; pkv_bm_swap_in gives it fresh blocks to copy back into with
 * kv_swap_in.
 *
 * Ordering with the GPU.  The manager only does bookkeeping on the host.  Blocks it
 * releases may be handed out by a later call, so the caller issues the kernels that read
 * them (kv_swap_out, or attention over a finished sequence) before any kernel that writes
 * blocks reserved by a later call, e.g. in order on one stream.
 *
 * Threads: every call locks the manager; calls from several threads are serialized.
 * Sequences are named by caller-chosen int64 ids.  Errors use the PKV_ERR_* codes of
 * pkv.h plus the two below; a failing call changes nothing.
 */
#ifndef PKV_BLOCK_MANAGER_H
#define PKV_BLOCK_MANAGER_H

#include <stdint.h>

#include "pkv.h"

#ifdef __cplusplus
extern "C" {
#endif

#define PKV_ERR_NO_BLOCKS  -10   /* not enough free (or evictable) blocks for the request */
#define PKV_ERR_STATE      -11   /* unknown / existing / swapped-out sequence, or a broken invariant */

typedef struct pkv_block_manager* pkv_bm_t;

typedef struct {
    int64_t num_blocks;        /* pool size                                         */
    int64_t free_blocks;       /* on the free list                                  */
    int64_t cached_blocks;     /* unreferenced but still in the prefix cache         */
    int64_t used_blocks;       /* referenced by at least one table                  */
    int64_t shared_blocks;     /* referenced by two or more tables                  */
    int64_t num_sequences;     /* live sequences, swapped-out ones included          */
    int64_t prefix_queries;    /* full prompt blocks looked up in the prefix cache   */
    int64_t prefix_hits;       /* of which found                                    */
    int64_t cow_copies;        /* copy-on-write pairs handed out                    */
    int64_t evictions;         /* cached blocks reclaimed for new allocations        */
} pkv_bm_stats;

/* A manager of blocks 0 .. num_blocks-1, all free.  enable_prefix_cache != 0 turns the
 * prefix cache on. */
PKV_API int pkv_bm_create(int32_t num_blocks, int enable_prefix_cache, pkv_bm_t* out);
PKV_API int pkv_bm_destroy(pkv_bm_t bm);

/* Blocks an allocation can take now: free plus evictable cached blocks (the pages'
 * free_blocks()).  Negative on error. */
PKV_API int64_t pkv_bm_free_blocks(pkv_bm_t bm);

/* References to `block` (tables holding it), or PKV_ERR_ARG for an id outside the pool. */
PKV_API int pkv_bm_refcount(pkv_bm_t bm, int32_t block);

/*
 * Start sequence seq_id with a prompt of n_prompt tokens (ids in prompt [host], or NULL
 * when they are not known; then nothing is looked up or cached for this sequence).
 * With the prefix cache on, the sequence attaches to the longest run of cached blocks
 * matching the prompt's first full blocks, at most floor((n_prompt - 1) / 16) of them;
 * *num_cached_tokens [host, may be NULL] receives 16 times that count.  The sequence's
 * length starts at that count of tokens: the caller appends the remaining prompt tokens
 * with pkv_bm_append_slots.  No block is allocated here.
 */
PKV_API int pkv_bm_add_sequence(pkv_bm_t bm, int64_t seq_id, const int32_t* prompt, int32_t n_prompt,
                                int32_t* num_cached_tokens);

/*
 * Blocks pkv_bm_append_slots(seq_id, n) would take from the pool: the new blocks the n
 * tokens reach plus one if the partly filled last block is shared.  Negative on error.
 */
PKV_API int pkv_bm_blocks_needed(pkv_bm_t bm, int64_t seq_id, int32_t n);

/*
 * Reserve slots for the sequence's next n tokens (positions len .. len+n-1), taking
 * blocks on demand.  slot_mapping [host] int32 [n] receives block * 16 + offset for each
 * token, ready for kv_append.  tokens [host] int32 [n] are the token ids (for the prefix
 * cache) or NULL.  If the partly filled last block is shared, it is first replaced by a
 * fresh private block: *cow_src / *cow_dst [host] receive the pair and *num_cow 1 (else
 * 0); the caller runs kv_copy_blocks(cow_src, cow_dst) before kv_append.  Blocks that
 * fill up with known tokens enter the prefix cache.  PKV_ERR_NO_BLOCKS if the pool cannot
 * supply pkv_bm_blocks_needed blocks (nothing changes).
 */
PKV_API int pkv_bm_append_slots(pkv_bm_t bm, int64_t seq_id, const int32_t* tokens, int32_t n,
                                int32_t* slot_mapping, int32_t* cow_src, int32_t* cow_dst, int32_t* num_cow);

/* New sequence child_id sharing every block of parent_id (same length and tokens). */
PKV_API int pkv_bm_fork(pkv_bm_t bm, int64_t parent_id, int64_t child_id);

/* End a sequence: release its blocks (last block first) and forget it. */
PKV_API int pkv_bm_free_sequence(pkv_bm_t bm, int64_t seq_id);

/*
 * Copy the block table of seq_id into table [host] int32 [capacity].  *num_blocks and
 * *num_tokens [host, may be NULL] receive its length in blocks and tokens.  A swapped-out
 * sequence has 0 blocks.  PKV_ERR_ARG (with the counts set) if capacity is too small.
 */
PKV_API int pkv_bm_block_table(pkv_bm_t bm, int64_t seq_id, int32_t* table, int32_t capacity, int32_t* num_blocks,
                               int32_t* num_tokens);

/*
 * Swap a sequence out: blocks [host] int32 [capacity] receives its table (the blocks to
 * copy to host slots 0 .. *num_blocks-1 with kv_swap_out), then the blocks are released
 * and the sequence is marked swapped out (it keeps its length and tokens).
 */
PKV_API int pkv_bm_swap_out(pkv_bm_t bm, int64_t seq_id, int32_t* blocks, int32_t capacity, int32_t* num_blocks);

/*
 * Swap a sequence back in: it gets *num_blocks fresh blocks, written to blocks [host]
 * int32 [capacity] in table order; the caller copies host slot j into blocks[j] with
 * kv_swap_in.  PKV_ERR_NO_BLOCKS if the pool cannot supply them.
 */
PKV_API int pkv_bm_swap_in(pkv_bm_t bm, int64_t seq_id, int32_t* blocks, int32_t capacity, int32_t* num_blocks);

PKV_API int pkv_bm_get_stats(pkv_bm_t bm, pkv_bm_stats* out);

/*
 * Verify the manager's invariants: each reference count equals the number of table
 * entries holding the block; every block is exactly one of free, cached-unreferenced or
 * referenced; a live sequence of len tokens holds ceil(len / 16) blocks (so at most its
 * last block is partly filled); prefix-cache entries point at blocks carrying their key.
 * PKV_OK or PKV_ERR_STATE.
 */
PKV_API int pkv_bm_check(pkv_bm_t bm);

#ifdef __cplusplus
}
#endif

#endif /* PKV_BLOCK_MANAGER_H */
