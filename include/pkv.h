/*
 * pkv.h — C ABI of the B200 paged KV-cache decode library (libpagedkv.so).
 *
 * Two operations make up one decode step of a vLLM-style serving loop:
 *
 *   reshape_and_cache       append each new token's K and V rows to the paged
 *                           cache at the slot the scheduler gave it
 *                           ("vLLM inference cost optimisation",
 *                           developer.aliyun.com, section 1: the decode loop
 *                           generates new K/V and writes them into the KV cache).
 *   paged_attention_decode  for every running sequence, the single new query of
 *                           each head attends over all cached tokens,
 *                           out = softmax(q K^T * scale) V (same article, section 2),
 *                           reading K/V block by block through the sequence's
 *                           block table, which maps logical blocks to scattered
 *                           physical blocks of a shared pool (same article,
 *                           section 4 "PagedAttention"; wzjinhao.cn vLLM
 *                           write-up, section 2.1).
 *
 * Layouts (row-major; the pages fix none of them):
 *   k_cache, v_cache   [num_blocks][num_kv_heads][block_size][head_dim]
 *                      elements of kv_dtype. One (block, kv head) tile is
 *                      block_size*head_dim elements, contiguous.
 *   q, out             [num_seqs][num_heads][head_dim], q_dtype (out has q's dtype).
 *   block_tables       int32 [num_seqs][max_blocks_per_seq]; entry j of row s
 *                      is the physical block of logical block j of sequence s.
 *                      Only entries j < ceil(seq_lens[s] / block_size) are read.
 *   seq_lens           int32 [num_seqs]: cached tokens to attend over,
 *                      including the token being decoded. 0 gives a zero row.
 *   k, v (append)      [num_tokens][num_kv_heads][head_dim] of in_dtype.
 *   slot_mapping       int64 [num_tokens]: slot = block * block_size + offset;
 *                      a negative slot writes nothing.
 * Grouped-query attention: query head g reads KV head g / (num_heads / num_kv_heads)
 * (a group of query heads shares one KV head: Aliyun article, GQA/MQA section).
 *
 * dtypes: q_dtype/kv_dtype pairs (F32, F32), (BF16, BF16), (BF16, FP8_E4M3),
 * (BF16, FP8_E5M2), (BF16, INT8); the append writes F32 or BF16 rows into any
 * of them (into a cache of another dtype only when it is an 8-bit one).
 * FP8 caches hold OCP E4M3 codes of x / scale with per-tensor fp32 scales
 * (Aliyun article, section 15 "the KV cache itself can be quantized";
 * promptx.wiki tutorial, per-tensor KV scales). Arithmetic is fp32 throughout.
 * head_dim in {64, 128}; block_size in {8, 16, 32};
 * num_heads / num_kv_heads in {1, 2, 4, 5, 8}.
 *
 * Ownership and synchronisation: every pointer except `stream` is DEVICE
 * memory owned by the caller. The library never allocates, never frees and
 * never synchronises; all work is enqueued on `stream` (a cudaStream_t, NULL =
 * the legacy default stream) and the calls return as soon as it is queued.
 *
 * Errors: problems visible on the host (null pointers, unsupported sizes or
 * dtypes, a workspace that is too small) return a non-zero pkv_status before
 * anything is launched. A failed launch returns PKV_ERR_LAUNCH. Bad DATA
 * (a block id outside [0, num_blocks), a seq_len outside
 * [0, max_blocks_per_seq * block_size], a slot past the end of the pool) is
 * never read or written: the kernels skip the access and OR one of the
 * PKV_DEVERR_* bits into a device error word, which the caller reads with
 * pkv_read_device_error().
 */
#ifndef PKV_H
#define PKV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PKV_API __attribute__((visibility("default")))
#else
#define PKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PKV_OK = 0,
    PKV_ERR_NULL = 1,        /* a required pointer is NULL */
    PKV_ERR_SHAPE = 2,       /* unsupported or inconsistent size */
    PKV_ERR_DTYPE = 3,       /* unsupported dtype or dtype pair */
    PKV_ERR_WORKSPACE = 4,   /* workspace missing or smaller than paged_attention_workspace_size() */
    PKV_ERR_LAUNCH = 5,      /* the CUDA runtime refused or failed the launch */
    PKV_ERR_DEVICE = 6       /* device query failed (no device, bad context) */
} pkv_status;

/* PKV_FP8_E5M2: OCP E5M2 codes (bias 15, largest finite 57344), per-tensor
 * scales like E4M3; decoded by the tensor-core kernel only (bf16 q, head_dim
 * 128, block 16 or 32); other shapes return PKV_ERR_SHAPE / PKV_ERR_DTYPE. */
/* PKV_INT8: symmetric 8-bit integer codes, code = clamp(round-half-even(x /
 * scale), -127, 127), value = code * scale; per-tensor or per-KV-head scales
 * like the FP8 formats, same shapes as PKV_FP8_E5M2. */
typedef enum { PKV_F32 = 0, PKV_BF16 = 1, PKV_FP8_E4M3 = 2, PKV_FP8_E5M2 = 3, PKV_INT8 = 4 } pkv_dtype;

/* Bits of the device error word. */
#define PKV_DEVERR_BLOCK_ID 1  /* a block-table entry outside [0, num_blocks): block skipped */
#define PKV_DEVERR_SEQ_LEN 2   /* seq_len < 0 or > max_blocks_per_seq * block_size: clamped */
#define PKV_DEVERR_SLOT 4      /* append slot >= num_blocks * block_size: row skipped */
#define PKV_DEVERR_TIMEOUT 8   /* a bounded pipeline wait gave up (output incomplete) */
#define PKV_DEVERR_PLAN 16     /* a shared-prefix plan entry out of range: that sequence's output is unspecified */

/*
 * Bytes of device workspace paged_attention_decode needs: a 256-byte header
 * (error word, work-claim counters), one arrival counter per (sequence, kv
 * head), one 8-byte completion stamp per work chunk (5 * num_partitions) and
 * fp32 split-KV partials (o[G][head_dim], m[G], l[G]) for up to
 * 4 * (5 * num_partitions) + num_seqs * num_kv_heads segments (a partition's
 * share of the work is cut into at most 5 chunks). num_partitions = 0 sizes it
 * for the automatic partition count on the current device. Returns 0 for
 * unsupported sizes.
 */
PKV_API size_t paged_attention_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                      int num_partitions);

/*
 * Zero a workspace (asynchronously on `stream`). Required once after the
 * workspace is allocated, and again after a call that reported
 * PKV_DEVERR_TIMEOUT or returned PKV_ERR_LAUNCH; every normal call leaves the
 * workspace's counters at zero.
 */
PKV_API int pkv_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/*
 * Paged decode attention. The total work, sum over (sequence, kv head) of
 * ceil(seq_len / block_size) blocks, taken in (sequence, kv head, block) order,
 * is shared between num_partitions CTAs (0 = one or more per SM, from the
 * occupancy); a piece of work may cover several (sequence, kv head) pairs and
 * a pair may be split between pieces. Each piece streams its K/V tiles through
 * shared memory and keeps an online softmax; no CTA ever waits for another. A
 * pair split between pieces leaves one fp32 partial (o, m, l) per piece in the
 * workspace, and the log-sum-exp merge of those partials writes its output.
 * Tensor-core kernel (bf16 and 8-bit caches of the shapes paged_decode_step
 * lists): every CTA takes an equal share of three quarters of the work, then
 * claims small chunks of the last quarter from a workspace counter until none
 * is left (the pieces are the same whichever CTA takes them, so the result
 * does not depend on timing); a second, small kernel launched right behind the
 * decode kernel on `stream` does the merge. CUDA-core kernel (F32 caches and
 * the other shapes): equal runs, and the run that finishes a pair last merges
 * it inside the same launch.
 *
 *   out          [num_seqs][num_heads][head_dim], q_dtype
 *   q            [num_seqs][num_heads][head_dim], q_dtype
 *   scale        softmax scale (1/sqrt(head_dim) for standard attention)
 *   k_scale, v_scale  per-tensor dequantisation scales for FP8 caches
 *                (ignored for F32/BF16 caches)
 *   workspace    device buffer of >= paged_attention_workspace_size(...,
 *                num_partitions) bytes, zeroed once by pkv_workspace_init;
 *                calls that share a workspace must not overlap on the GPU.
 */
PKV_API int paged_attention_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, const int32_t* seq_lens, int num_seqs,
                           int num_heads, int num_kv_heads, int head_dim, int block_size, float scale,
                           int max_blocks_per_seq, int num_blocks, int q_dtype, int kv_dtype,
                           float k_scale, float v_scale, int num_partitions,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * One whole decode step: the append of each sequence's new token (reshape_and_cache of
 * new_k/new_v row s at slot_mapping[s], one new token per sequence) followed by
 * paged_attention_decode over the cache that includes it. For bf16 and 8-bit caches of
 * the shapes the tensor-core decode kernel covers (block_size 16 or 32, group <= 8,
 * head_dim 64/128 for bf16, 128 for E4M3, E5M2 and INT8) both happen in ONE launch: the warp that
 * streams a sequence's last block first writes the new rows into it. Other shapes run
 * the two calls in stream order. Results are those of the two calls.
 *
 *   new_k, new_v   [num_seqs][num_kv_heads][head_dim] of in_dtype (F32 or BF16)
 *   slot_mapping   int64 [num_seqs]; a non-negative slot must lie in the block that
 *                  holds position seq_lens[s] - 1 of sequence s (its last block), so
 *                  seq_lens[s] >= 1; a negative slot appends nothing.
 * Other arguments as paged_attention_decode; slot errors go to the workspace error word.
 * The one-launch form raises PKV_DEVERR_SLOT for a slot outside the last block (still
 * written, but sequence s's output is then unspecified) and for a non-negative slot of
 * a sequence with seq_lens[s] == 0 (nothing written).
 */
PKV_API int paged_decode_step(void* out, const void* q, void* k_cache, void* v_cache, const int32_t* block_tables,
                              const int32_t* seq_lens, int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                              int block_size, float scale, int max_blocks_per_seq, int num_blocks, int q_dtype,
                              int kv_dtype, float k_scale, float v_scale, int num_partitions, void* workspace,
                              size_t workspace_bytes, const void* new_k, const void* new_v,
                              const int64_t* slot_mapping, int in_dtype, void* stream);

/*
 * FP8 caches with one scale per KV head (the promptx.wiki inference tutorial,
 * quantisation section, sets per-tensor against per-attention-head KV
 * quantisation): k_head_scales / v_head_scales are device arrays of
 * num_kv_heads floats > 0 (caller-owned, read during the call), used where the
 * per-tensor calls use k_scale / v_scale — the append encodes
 * code = FP8(x / k_head_scales[h]) for KV head h, the decode dequantises with
 * the same scale. kv_dtype must be FP8_E4M3, FP8_E5M2 or INT8; the decode runs on
 * the tensor-core kernel only (the shapes paged_attention_decode lists for
 * it), others return PKV_ERR_SHAPE; a null scale array returns PKV_ERR_NULL.
 * Otherwise the same as reshape_and_cache and paged_attention_decode.
 */
PKV_API int reshape_and_cache_head_scales(const void* k, const void* v, void* k_cache, void* v_cache,
                                          const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                                          int head_dim, int block_size, int num_blocks, int in_dtype, int kv_dtype,
                                          const float* k_head_scales, const float* v_head_scales,
                                          int32_t* device_error, void* stream);
PKV_API int paged_attention_decode_head_scales(void* out, const void* q, const void* k_cache, const void* v_cache,
                                               const int32_t* block_tables, const int32_t* seq_lens, int num_seqs,
                                               int num_heads, int num_kv_heads, int head_dim, int block_size,
                                               float scale, int max_blocks_per_seq, int num_blocks, int q_dtype,
                                               int kv_dtype, const float* k_head_scales,
                                               const float* v_head_scales, int num_partitions, void* workspace,
                                               size_t workspace_bytes, void* stream);

/*
 * Several new tokens per sequence (chunked prefill, speculative-decoding
 * verification): q_len queries per sequence, causal within the chunk. Query j
 * of sequence s is the token at position seq_lens[s] - q_len + j (seq_lens
 * counts the q_len new tokens, already appended with reshape_and_cache) and
 * attends the cached tokens 0 .. seq_lens[s] - q_len + j, i.e. all earlier
 * tokens and itself; a query whose position is negative gets a zero row.
 *
 *   q, out       [num_seqs][q_len][num_heads][head_dim], q_dtype BF16
 *   q_len        1 .. 8 with q_len * (num_heads / num_kv_heads) in {1, 2, 4, 5, 8}
 *   workspace    >= paged_attention_workspace_size(num_seqs, q_len * num_heads,
 *                num_kv_heads, head_dim, num_partitions) bytes
 * Other arguments as paged_attention_decode. Runs on the tensor-core kernel
 * (bf16 / E4M3 / E5M2 / INT8 caches, block size 16 or 32, head_dim 128, or 64 for
 * bf16); other shapes return PKV_ERR_SHAPE. q_len = 1 is paged_attention_decode.
 */
PKV_API int paged_attention_decode_mq(void* out, const void* q, const void* k_cache, const void* v_cache,
                                      const int32_t* block_tables, const int32_t* seq_lens, int num_seqs,
                                      int q_len, int num_heads, int num_kv_heads, int head_dim, int block_size,
                                      float scale, int max_blocks_per_seq, int num_blocks, int q_dtype,
                                      int kv_dtype, float k_scale, float v_scale, int num_partitions,
                                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * Shared-prefix decode. Prefix caching reuses whole blocks: sequences whose
 * tables hold the same physical block hold the same tokens there (wzjinhao.cn
 * vLLM write-up, section 2.3 "Chunked Prefill and Prefix Caching";
 * "vLLM inference cost optimisation", section 11). Given a plan of such
 * sharing (pkv_prefix_plan in pkv_blocks.h, on the same tables), this call
 * reads every shared block once for all the sequences of its group: a prefix
 * pass attends the queries of up to max_group members (max_group *
 * num_heads / num_kv_heads <= 32 query columns per KV head) against each
 * shared block, each member seeing only its own shared blocks; a suffix pass
 * attends each sequence over the rest of its table; a merge combines the two
 * by their log-sum-exp weights. The output equals paged_attention_decode's
 * (same softmax over the same tokens, up to the order of the fp32 sums).
 *
 * The plan (device arrays, caller-owned, pkv_prefix_plan's outputs):
 *   group_members  int32, members of group g at [group_offsets[g], group_offsets[g + 1])
 *   group_offsets  int32 [num_groups + 1]
 *   group_tables   int32 [num_groups][max_blocks_per_seq]: row g = the group's shared blocks
 *   group_lens     int32 [num_groups]: tokens in row g (its blocks x block_size)
 *   shared_blocks  int32 [num_seqs]: leading (full) blocks of sequence s read through its
 *                  group's row; > 0 only for members of a group
 *   num_groups     0 .. num_seqs (0: the plain decode, bit for bit)
 * Tensor-core shapes only (bf16 q; bf16, E4M3, E5M2 or INT8 caches; block 16 or
 * 32; head_dim 128, or 64 for bf16); no per-head scales, one query per sequence.
 * workspace >= paged_attention_shared_prefix_workspace_size(num_seqs, num_heads,
 * num_kv_heads, head_dim, num_groups, num_partitions) bytes, zeroed once.
 * Errors: host checks as paged_attention_decode (PKV_ERR_SHAPE also for
 * max_group * num_heads / num_kv_heads > 32); a group with more than max_group
 * members, a member index outside [0, num_seqs) or a shared count beyond a
 * sequence's full blocks or its group's row sets PKV_DEVERR_PLAN, and the
 * outputs of the sequences concerned are unspecified. Launches: the prefix pass
 * (when num_groups > 0), the suffix pass and the merge, in order on `stream`.
 */
PKV_API size_t paged_attention_shared_prefix_workspace_size(int num_seqs, int num_heads, int num_kv_heads,
                                                            int head_dim, int num_groups, int num_partitions);
PKV_API int paged_attention_decode_shared_prefix(void* out, const void* q, const void* k_cache, const void* v_cache,
                                                 const int32_t* block_tables, const int32_t* seq_lens, int num_seqs,
                                                 int num_heads, int num_kv_heads, int head_dim, int block_size,
                                                 float scale, int max_blocks_per_seq, int num_blocks, int q_dtype,
                                                 int kv_dtype, float k_scale, float v_scale,
                                                 const int32_t* group_members, const int32_t* group_offsets,
                                                 const int32_t* group_tables, const int32_t* group_lens,
                                                 const int32_t* shared_blocks, int num_groups, int max_group,
                                                 int num_partitions, void* workspace, size_t workspace_bytes,
                                                 void* stream);
/*
 * The decode step of paged_decode_step with the shared-prefix decode: the append
 * of each sequence's new token rides in the suffix pass's launch (the block
 * holding position seq_lens[s] - 1 must be the sequence's own, i.e. past its
 * shared blocks; otherwise PKV_DEVERR_SLOT). Arguments as
 * paged_attention_decode_shared_prefix plus those of paged_decode_step.
 */
PKV_API int paged_decode_step_shared_prefix(void* out, const void* q, void* k_cache, void* v_cache,
                                            const int32_t* block_tables, const int32_t* seq_lens, int num_seqs,
                                            int num_heads, int num_kv_heads, int head_dim, int block_size,
                                            float scale, int max_blocks_per_seq, int num_blocks, int q_dtype,
                                            int kv_dtype, float k_scale, float v_scale,
                                            const int32_t* group_members, const int32_t* group_offsets,
                                            const int32_t* group_tables, const int32_t* group_lens,
                                            const int32_t* shared_blocks, int num_groups, int max_group,
                                            int num_partitions, void* workspace, size_t workspace_bytes,
                                            const void* new_k, const void* new_v, const int64_t* slot_mapping,
                                            int in_dtype, void* stream);

/*
 * Test hook for the failure path (no counterpart in the pages). The same call
 * as paged_attention_decode, except that the producer warp that owns unit
 * `withheld_unit` (units = (sequence, KV-head group, block) in order) never
 * hands that unit's stage to its consumer warps and issues nothing after it.
 * The consumers' bounded wait (about one second) runs out, the launch sets
 * PKV_DEVERR_TIMEOUT in the workspace error word and returns; nothing faults or
 * hangs and the CUDA context stays usable. The output of that CTA's streams is
 * incomplete, and the workspace must be re-initialised (pkv_workspace_init)
 * before its next use. Only the tensor-core kernel has the hook: bf16 q with
 * bf16 or E4M3 caches of block size 16 or 32; other shapes return
 * PKV_ERR_SHAPE, as does withheld_unit < 0.
 */
PKV_API int pkv_test_decode_timeout(void* out, const void* q, const void* k_cache, const void* v_cache,
                                    const int32_t* block_tables, const int32_t* seq_lens, int num_seqs,
                                    int num_heads, int num_kv_heads, int head_dim, int block_size, float scale,
                                    int max_blocks_per_seq, int num_blocks, int q_dtype, int kv_dtype,
                                    float k_scale, float v_scale, int num_partitions, void* workspace,
                                    size_t workspace_bytes, int withheld_unit, void* stream);

/*
 * paged_attention_decode without a caller workspace, for callers that cannot
 * allocate device memory: plug-ins and custom operators whose host framework
 * owns every allocation and forbids allocating while they run, hosts that
 * reserve all device memory at start-up, and latency-bound serving loops that
 * cannot afford cudaMalloc's implicit device synchronisation. (The pages have
 * no counterpart; this is an interface convenience, same arithmetic as
 * paged_attention_decode.)
 *
 * Arguments are those of paged_attention_decode minus the workspace. The
 * scratch is a fixed 32 MiB array inside the library, present on every GPU
 * that loads it until the process exits; a call whose
 * paged_attention_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim,
 * num_partitions) exceeds 32 MiB returns PKV_ERR_WORKSPACE without launching.
 * Nothing is allocated. The first call on each device looks up the array's
 * device address (with that device current), so make that first call before
 * any stream capture; the address is looked up again when the device's
 * context changes (for instance after cudaDeviceReset). The call runs every
 * host check of paged_attention_decode before it queues anything; then it
 * clears the array's counters and error word on `stream` and launches. Every
 * call shares the array: calls that overlap on the GPU (other streams, other
 * threads) race and must be serialised by the caller. The device error word
 * is not readable through this entry point.
 */
PKV_API int paged_attention_decode_static(void* out, const void* q, const void* k_cache, const void* v_cache,
                                          const int32_t* block_tables, const int32_t* seq_lens, int num_seqs,
                                          int num_heads, int num_kv_heads, int head_dim, int block_size,
                                          float scale, int max_blocks_per_seq, int num_blocks, int q_dtype,
                                          int kv_dtype, float k_scale, float v_scale, int num_partitions,
                                          void* stream);

/*
 * Decode-step append: for every token t with slot_mapping[t] >= 0, write
 * k[t][h][:] to k_cache[slot / block_size][h][slot % block_size][:] (and v the
 * same way) for every kv head h. Same dtype: a bit copy. FP8_E4M3 cache from
 * F32 or BF16 rows: code = E4M3(x / k_scale) with an IEEE fp32 division and
 * round-to-nearest-even, saturating to +-448 (v with v_scale); FP8_E5M2 the
 * same with E5M2 codes, saturating to +-57344; INT8 code =
 * clamp(round-half-even(x / scale), -127, 127), NaN -> 0.
 * Duplicate non-negative slots in one call give an unspecified winner.
 * device_error: optional int32 device word that receives PKV_DEVERR_SLOT.
 */
PKV_API int reshape_and_cache(const void* k, const void* v, void* k_cache, void* v_cache,
                      const int64_t* slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                      int block_size, int num_blocks, int in_dtype, int kv_dtype,
                      float k_scale, float v_scale, int32_t* device_error, void* stream);

/*
 * Copy the workspace's device error word to *host_error (synchronising on
 * `stream`); clear != 0 also resets it to zero.
 */
PKV_API int pkv_read_device_error(void* workspace, size_t workspace_bytes, int32_t* host_error, int clear,
                          void* stream);

/*
 * Host check of a decode batch's tables before they go to the device (host
 * buffers, caller-owned; no device access). The kernels catch the same cases
 * on the device and report them in the workspace error word; this call lets a
 * scheduler find them first. Checks, per sequence s, the rules of the layouts
 * above: seq_lens[s] in [0, max_blocks_per_seq * block_size] (else
 * PKV_DEVERR_SEQ_LEN), entries j < ceil(seq_lens[s] / block_size) of row s in
 * [0, num_blocks) (else PKV_DEVERR_BLOCK_ID), and, when slot_mapping is given
 * (int64 [num_seqs], one new token per sequence as paged_decode_step takes
 * it), every non-negative slot below num_blocks * block_size, inside the block
 * that holds position seq_lens[s] - 1 and not also another sequence's slot
 * (else PKV_DEVERR_SLOT). *bad_bits = the PKV_DEVERR_* bits found (0: clean),
 * *first_bad = the first sequence with a problem or -1. Returns PKV_OK,
 * PKV_ERR_NULL, PKV_ERR_SHAPE (num_seqs < 0, a size <= 0) or PKV_BM_HOST_ALLOC
 * (host memory exhausted).
 */
PKV_API int pkv_validate_tables(const int32_t* block_tables, const int32_t* seq_lens, int num_seqs,
                                int max_blocks_per_seq, int block_size, int num_blocks,
                                const int64_t* slot_mapping, int32_t* bad_bits, int32_t* first_bad);

/* Number of partitions num_partitions = 0 resolves to for this configuration on the current device. */
PKV_API int pkv_default_partitions(int head_dim, int block_size, int num_heads, int num_kv_heads, int kv_dtype);

/*
 * Kernel for decodes of FP8 (E4M3 / E5M2) caches, process-wide:
 *   PKV_FP8_KERNEL_MMA (0, the default): warp-level tensor-core products on codes widened
 *     exactly to f16 (every FP8 shape the library covers);
 *   PKV_FP8_KERNEL_TCGEN05 (1): fifth-generation tensor cores (tcgen05.mma, accumulators in
 *     tensor memory) reading the 8-bit K and V tiles as they lie, for head_dim 128, block size 16
 *     or 32 and a multiple of 128 / block_size KV heads; other FP8 shapes keep the default
 *     kernel. Same results within the FP8 tolerance; on the measured workloads it is slower
 *     than the default.
 * Applies to calls queued after it (plain and fused decode steps, several new tokens per
 * sequence, per-head scales and the no-allocation entry point; the shared-prefix passes always
 * use the default). Returns the previous choice, or -PKV_ERR_SHAPE for an unknown value.
 */
#define PKV_FP8_KERNEL_MMA 0
#define PKV_FP8_KERNEL_TCGEN05 1
PKV_API int pkv_set_fp8_kernel(int which);

/* Static description of a status code. */
PKV_API const char* pkv_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H */
