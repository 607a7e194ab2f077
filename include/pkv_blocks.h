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
#define PKV_BM_HOST_ALLOC 24  /* a host allocation failed (the call may have been partly applied) */

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

/*
 * Shared-prefix plan of one decode batch (host buffers in, host buffers out,
 * all caller-owned; no device access). The pages' prefix caching reuses whole
 * blocks (wzjinhao.cn vLLM write-up, section 2.3; "vLLM inference cost
 * optimisation", section 11): sequences whose tables hold the same physical
 * block hold the same tokens there, so one pass over that block can serve the
 * queries of all of them. This call finds those blocks; the decode of a group
 * then reads each one once and merges it with every member's own remainder.
 *
 * Rule (a reading; the pages give no grouping procedure): only full blocks
 * count (block j of sequence s when (j + 1) * block_size <= seq_lens[s] and
 * the entry is >= 0). Candidates are the sequences whose first block is full,
 * bucketed by its id (buckets in order of their first sequence), each bucket
 * cut into chunks of max_group sequences in index order; a chunk of one stays
 * alone. In a chunk, for j = 0, 1, ...: among the members still sharing, take
 * the id that most of them hold at j (ties: the first such member's id); stop
 * when no id is held by two; the members holding it keep sharing.
 *
 *   block_tables   int32 [num_seqs][max_blocks_per_seq], -1 padded (the decode's tables)
 *   seq_lens       int32 [num_seqs]
 *   group_members  int32 [num_seqs]   out: member sequence indices, group after group
 *   group_offsets  int32 [num_seqs + 1] out: group g = members [offsets[g], offsets[g + 1])
 *   group_tables   int32 [num_seqs][max_blocks_per_seq] out: row g = the group's shared
 *                  blocks, -1 padded (rows >= *num_groups untouched)
 *   group_lens     int32 [num_seqs]   out: tokens in row g's blocks (blocks x block_size)
 *   shared_blocks  int32 [num_seqs]   out: leading blocks of sequence s read through its
 *                  group's row (they equal its own table's); 0 = outside every group
 * Returns PKV_OK, PKV_ERR_NULL, or PKV_ERR_SHAPE (num_seqs < 0, a size <= 0 or
 * max_group < 1). max_group 1 makes no groups.
 */
PKV_API int pkv_prefix_plan(const int32_t* block_tables, const int32_t* seq_lens, int num_seqs,
                            int max_blocks_per_seq, int block_size, int max_group, int32_t* group_members,
                            int32_t* group_offsets, int32_t* group_tables, int32_t* group_lens,
                            int32_t* shared_blocks, int* num_groups);

/*
 * Inputs of the two passes of a shared-prefix decode, from a pkv_prefix_plan result (host
 * buffers, caller-owned). The prefix pass runs over the plan's group rows with 8 query
 * columns per KV head: member i of group g takes columns i * Gq .. i * Gq + Gq - 1
 * (Gq = query heads per KV head) and sees its own shared blocks only; the suffix pass runs
 * every sequence over the rest of its own table.
 *
 *   col_seq       int32 [num_groups][8] out: sequence of each column, -1 = unused
 *   col_limit     int32 [num_groups][8] out: tokens that column sees (shared blocks x block_size)
 *   suffix_tables int32 [num_seqs][max_blocks_per_seq] out: row s = block_tables[s] shifted left
 *                 by shared_blocks[s], -1 padded
 *   suffix_lens   int32 [num_seqs] out: seq_lens[s] - shared_blocks[s] * block_size
 * Returns PKV_OK, PKV_ERR_NULL, or PKV_ERR_SHAPE (a group with more than 8 / Gq members,
 * Gq not dividing 8, a shared count beyond the table or the length, bad sizes).
 */
PKV_API int pkv_prefix_pass_inputs(const int32_t* block_tables, const int32_t* seq_lens, int num_seqs,
                                   int max_blocks_per_seq, int block_size, const int32_t* group_members,
                                   const int32_t* group_offsets, int num_groups, const int32_t* shared_blocks,
                                   int query_heads_per_kv_head, int32_t* col_seq, int32_t* col_limit,
                                   int32_t* suffix_tables, int32_t* suffix_lens);

#ifdef __cplusplus
}
#endif
