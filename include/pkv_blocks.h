/*
 * pkv_blocks.h — host-side block manager for the paged KV cache: the pool of
 * physical blocks, each sequence's block table, reference counts for blocks
 * shared between sequences, and the slot of every new token.
 *
 * What it restates ("vLLM inference cost optimisation", developer.aliyun.com,
 * section 4 and 4.1; wzjinhao.cn vLLM write-up, sections 2.1 and 2.3): the KV
 * cache is a pool of fixed-size blocks (block_size tokens of every KV head); a
 * sequence's block table maps its logical block i to a physical block, so a
 * sequence's cache is logically contiguous and physically scattered, and a
 * block is allocated only when the previous one is full. Sequences that share
 * a prefix share its whole blocks. The pages describe the pool and the table
 * but no allocator; the policy below is this library's reading:
 *
 *  - Free list: a FIFO queue, initially 0, 1, ..., num_blocks-1. Allocation
 *    takes the front; a block whose reference count drops to 0 goes to the back.
 *  - Fork: the child's table is a copy of the parent's, every block's count +1.
 *  - Append (one new token at position L = current length): if L % block_size
 *    is 0 a new block is allocated and added to the table; otherwise the new
 *    token lands in the last block, and if that block is shared (count > 1) it
 *    is first copied ("copy on write"): a new block replaces it in this
 *    sequence's table, the old block's count drops by 1, and the pair
 *    (old, new) is reported so the caller copies the block's rows on the GPU
 *    before the step's reshape_and_cache. slot = table[L / bs] * bs + L % bs.
 *  - Free: every block's count -1; blocks reaching 0 return to the free list
 *    in table order.
 * Calls that need a block when none is free fail with PKV_BM_NO_BLOCKS and
 * change nothing (pkv_bm_step: the sequences before the failing one keep
 * their append, see below). Not thread-safe: one manager per scheduler thread.
 * (The pages have no counterpart for this interface; it is plumbing for the
 * decode step's block_tables / seq_lens / slot_mapping.)
 */
#pragma once

#include <stdint.h>

#include "pkv.h"

#ifdef __cplusplus
extern "C" {
#endif

/* extra status codes (pkv_status values 0..6 keep their meaning) */
#define PKV_BM_NO_BLOCKS 20   /* the pool has no free block for this request */
#define PKV_BM_UNKNOWN_SEQ 21 /* no sequence with this id */
#define PKV_BM_DUPLICATE_SEQ 22
#define PKV_BM_TABLE_FULL 23  /* the sequence would need more than max_blocks_per_seq blocks */

typedef struct pkv_block_manager pkv_block_manager;

/* A manager over blocks 0..num_blocks-1; NULL for sizes <= 0 or allocation failure. Host memory only. */
PKV_API pkv_block_manager* pkv_bm_create(int num_blocks, int block_size, int max_blocks_per_seq);
PKV_API void pkv_bm_destroy(pkv_block_manager* bm);

/* New sequence holding prompt_len tokens (ceil(prompt_len / block_size) fresh blocks). */
PKV_API int pkv_bm_add(pkv_block_manager* bm, int64_t seq_id, int prompt_len);
/* child shares every block of parent (same length). */
PKV_API int pkv_bm_fork(pkv_block_manager* bm, int64_t parent_id, int64_t child_id);
/* Reserve the slot of one new token of seq_id; *cow_src / *cow_dst = the copied block pair, or -1. */
PKV_API int pkv_bm_append(pkv_block_manager* bm, int64_t seq_id, int64_t* slot, int32_t* cow_src, int32_t* cow_dst);
PKV_API int pkv_bm_free(pkv_block_manager* bm, int64_t seq_id);

PKV_API int pkv_bm_num_free(const pkv_block_manager* bm);
/* Current length of seq_id, or -1 if unknown. */
PKV_API int pkv_bm_seq_len(const pkv_block_manager* bm, int64_t seq_id);
/* Reference count of a block (0 = free), or -1 for an id outside the pool. */
PKV_API int pkv_bm_ref_count(const pkv_block_manager* bm, int block);

/*
 * One decode step for n sequences, in order: append one token to each, then
 * write the decode inputs (host buffers, caller-owned):
 *   slot_mapping  int64 [n]            the new token's slot
 *   block_tables  int32 [n][max_blocks_per_seq], padded with -1
 *   seq_lens      int32 [n]            lengths after the append
 *   cow_pairs     int32 [2 * n]        (src, dst) block pairs to copy before the append writes,
 *                                      *n_cow of them (at most one per sequence)
 * On PKV_BM_NO_BLOCKS (or another error) at sequence i, *n_done = i: sequences
 * 0..i-1 were appended (their slot_mapping and cow pairs are written) and the
 * tables are not; the caller frees or preempts and retries the rest.
 */
PKV_API int pkv_bm_step(pkv_block_manager* bm, const int64_t* seq_ids, int n, int64_t* slot_mapping,
                        int32_t* block_tables, int32_t* seq_lens, int32_t* cow_pairs, int* n_cow, int* n_done);

/* Tables and lengths of n sequences without appending (same layout as pkv_bm_step). */
PKV_API int pkv_bm_tables(const pkv_block_manager* bm, const int64_t* seq_ids, int n, int32_t* block_tables,
                          int32_t* seq_lens);

#ifdef __cplusplus
}
#endif
