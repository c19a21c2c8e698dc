/*
 * pa_block_manager.h -- host-side KV block manager of libpagedattn.so.
 *
 * Decides where every token's K/V lives in a pool of fixed-size physical
 * blocks and produces what the kernels of pa_api.h consume: slots for
 * pa_append_kv, block tables and lengths for pa_decode*, and (src, dst)
 * pairs for pa_copy_blocks. Host memory only; no CUDA calls.
 *
 * What it follows (page titles and sections):
 *  - KV cache article (ainews.alishangtian.com), section
 *    "PagedAttention：把操作系统的老智慧搬进推理引擎": the cache of a request is
 *    cut into fixed-size blocks mapped by a block table; blocks are allocated
 *    on demand, so waste is limited to each request's last block; a prefix
 *    several requests share is stored once and reference-counted; branches
 *    copy a block only at the fork point (copy-on-write).
 *  - "AI 陪读顶会论文（三）：KV Cache 显存占用计算与 PagedAttention 原理拆解",
 *    section "PagedAttention 的破局哲学": a new block is taken only when token
 *    BS+1 (2*BS+1, ...) arrives; branches share prompt blocks until they
 *    diverge.
 *  - "第2章 KV Cache：模型内部的显存复用" (chapter overview): a radix tree
 *    organises the prefixes of multi-turn conversations so later requests hit
 *    the cached prefix. Here the tree is block-granular: each edge is one full
 *    block of token ids, because only whole physical blocks can be shared.
 *
 * Threading: a manager is not thread-safe; one host thread drives it.
 * Errors: functions return PA_BM_OK (0) or a negative PA_BM_ERR_* code and
 * leave the manager unchanged on error.
 */
#ifndef PA_BLOCK_MANAGER_H
#define PA_BLOCK_MANAGER_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PA_BM_OK 0
#define PA_BM_ERR_INVALID -1    /* bad argument, unknown or duplicate sequence id */
#define PA_BM_ERR_NO_BLOCKS -2  /* the pool (after evicting cached blocks) is exhausted */
#define PA_BM_ERR_CAPACITY -3   /* an output array is too small */

typedef struct pa_block_manager pa_block_manager;

/* A pool of num_blocks physical blocks of block_size tokens.
 * prefix_cache != 0 keeps full blocks of finished sequences in a radix tree
 * of token ids for reuse (evicted least-recently-used first when the free
 * list runs dry). Returns NULL on bad arguments or allocation failure. */
pa_block_manager* pa_bm_create(int64_t num_blocks, int32_t block_size, int32_t prefix_cache);
void pa_bm_destroy(pa_block_manager* bm);

/* Blocks on the free list, and blocks that only the prefix cache holds
 * (reclaimable). */
int64_t pa_bm_num_free_blocks(const pa_block_manager* bm);
int64_t pa_bm_num_cached_blocks(const pa_block_manager* bm);
/* Reference count of a physical block (number of sequences using it, plus
 * one while it is in the prefix cache); -1 for an id out of range. */
int32_t pa_bm_block_refcount(const pa_block_manager* bm, int64_t block);

/* Start sequence `seq_id` with the n_tokens prompt token ids `tokens`. With
 * the prefix cache on, the longest run of leading full blocks whose token ids
 * are cached is reused (shared, not copied); blocks for the rest of the
 * prompt are allocated. *cached_tokens receives how many leading prompt
 * tokens already have their K/V in the cache (a multiple of block_size); the
 * caller appends K/V for the others (pa_bm_slots gives their slots). */
int32_t pa_bm_add_sequence(pa_block_manager* bm, int64_t seq_id, const int32_t* tokens,
                           int32_t n_tokens, int32_t* cached_tokens);

/* Reserve the slot of the next token (position = current length) of a
 * sequence and return it in *slot. A new block is taken when the last one is
 * full. When the last block is partially filled and shared (after a fork),
 * the sequence gets a private block instead and *cow_src / *cow_dst receive
 * the block to copy (apply with pa_copy_blocks before appending); otherwise
 * both are -1. `token` is the token id, kept for the prefix cache. */
int32_t pa_bm_append_token(pa_block_manager* bm, int64_t seq_id, int32_t token, int64_t* slot,
                           int32_t* cow_src, int32_t* cow_dst);

/* pa_bm_append_token for a batch: one token (tokens[i]) for each of the n
 * distinct sequences seq_ids[i], in order, in one call. slots[n] receives
 * each token's slot; the copy-on-write pairs the batch needs, in order, go
 * to cow_pairs ([n][2] int32 (src, dst), room for n pairs) and their count to
 * *num_pairs; apply them (pa_copy_blocks) before appending K/V. A sequence
 * that copies drops its share of the old block, so a later sequence of the
 * batch that shared it with that one alone writes in place. The batch's
 * blocks are all taken before any of its tokens joins the prefix cache, so
 * when the pool must evict cached blocks the choice can differ from n
 * separate pa_bm_append_token calls (both placements are valid). Returns
 * PA_BM_ERR_INVALID for an unknown or repeated id and PA_BM_ERR_NO_BLOCKS if
 * the pool (after evicting cached blocks) cannot supply the batch; either
 * way nothing has changed. */
int32_t pa_bm_append_tokens(pa_block_manager* bm, const int64_t* seq_ids, const int32_t* tokens,
                            int32_t n, int64_t* slots, int32_t* cow_pairs, int32_t* num_pairs);

/* child_id starts as a copy of parent_id that shares all its blocks. */
int32_t pa_bm_fork(pa_block_manager* bm, int64_t parent_id, int64_t child_id);

/* End a sequence: its references are dropped; blocks nobody uses return to
 * the free list, or stay in the prefix cache if they are cached full blocks. */
int32_t pa_bm_free_sequence(pa_block_manager* bm, int64_t seq_id);

/* Sliding window support: release the blocks of a sequence that hold only
 * tokens before `position` (their table entries keep their old values, which
 * pa_decode_sliding_window never reads). */
int32_t pa_bm_release_before(pa_block_manager* bm, int64_t seq_id, int32_t position);

/* pa_bm_release_before(seq, length - window) for each of n sequences in one
 * call: after a step of sliding-window decoding (window >= 1 tokens, the
 * newest included), release the blocks that hold only tokens the window has
 * left behind. PA_BM_ERR_INVALID (nothing released) for an unknown id. */
int32_t pa_bm_release_window(pa_block_manager* bm, const int64_t* seq_ids, int32_t n,
                             int32_t window);

int32_t pa_bm_sequence_length(const pa_block_manager* bm, int64_t seq_id);

/* Slots of positions [first, first + count) of a sequence. */
int32_t pa_bm_slots(const pa_block_manager* bm, int64_t seq_id, int32_t first, int32_t count,
                    int64_t* slots);

/* Block tables [n_seqs][max_blocks_per_seq] (unused entries 0) and lengths
 * [n_seqs] of a batch, in the layout pa_decode reads. */
int32_t pa_bm_block_tables(const pa_block_manager* bm, const int64_t* seq_ids, int32_t n_seqs,
                           int32_t max_blocks_per_seq, int32_t* block_tables,
                           int32_t* context_lens);

/* Incremental form of pa_bm_block_tables for a caller that keeps the same
 * arrays from step to step: only the rows whose block list changed since
 * this call last wrote them are rewritten (a new block, a copy-on-write
 * replacement, or another sequence in the row); every length is written.
 * row_versions [n_seqs] (caller-owned, read and written) holds the stamp of
 * the table each row holds; stamps are never 0 and unique across the
 * manager's sequences, so zero-filled row_versions make the first call write
 * every row, and moving sequences between rows needs no reset. Reset
 * row_versions to 0 after writing the arrays by other means or changing
 * max_blocks_per_seq. *rows_written (may be NULL) receives the number of
 * rows rewritten. Errors as pa_bm_block_tables, with nothing written. */
int32_t pa_bm_block_tables_update(const pa_block_manager* bm, const int64_t* seq_ids,
                                  int32_t n_seqs, int32_t max_blocks_per_seq,
                                  int32_t* block_tables, int32_t* context_lens,
                                  uint64_t* row_versions, int32_t* rows_written);

#ifdef __cplusplus
}
#endif

#endif /* PA_BLOCK_MANAGER_H */
