// Internal declarations shared by the translation units of libpagedkv.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "pkv.h"

namespace pkv {

constexpr int kMaxSmemPerBlock = 227 * 1024;
constexpr int kMaxSeqs = 16384;         // per call: the per-sequence tile prefix lives in shared memory
constexpr int kMaxRunsPerSM = 3;        // automatic partition count is at most 3 runs per SM
constexpr size_t kWorkspaceHeader = 256;
constexpr int kMaxHeadGroup = 4;        // KV heads per MMA work unit (partial slots reserved per run)
// Tensor-core kernels: a CTA's first chunk is its share of three quarters of the work; the last
// quarter is cut into up to kTailChunksPerRun chunks per CTA, claimed as CTAs run dry. The
// workspace keeps partial slots for (1 + kTailChunksPerRun) chunks per run.
constexpr int kTailChunksPerRun = 4;
constexpr int kMinTailChunk = 16;       // units
// below this many units per CTA the split stays static: there a CTA's whole run lasts only some
// tens of microseconds, and tail chunks (and the merging of the extra pieces they cut) cost more
// than the imbalance they remove (measured on the long-context and Llama-3-8B-layer workloads)
constexpr int kMinUnitsForTail = 256;
constexpr float kLog2e = 1.4426950408889634074f;

struct DecodeParams {
    void* out;
    const void* q;
    const uint8_t* k_cache;
    const uint8_t* v_cache;
    const int32_t* block_tables;
    const int32_t* seq_lens;
    int num_seqs;
    int num_heads;
    int num_kv_heads;
    int max_blocks_per_seq;
    int num_blocks;
    float scale;       // softmax scale as given
    float k_scale;     // per-tensor dequantisation scales (1 for bf16 / f32 caches)
    float v_scale_in;
    float q_scale;     // set by the launcher: factor applied to q.K to get log2-domain scores
    float v_scale;     // set by the launcher: factor applied to the output
    int32_t* err;      // workspace error word
    int32_t* counters; // [num_seqs * num_kv_heads] arrivals, zero between calls
    float* partials;   // [(runs + pairs)][slot_floats]
    int slot_floats;
    int stages_per_warp; // set by the launcher
    // fused decode-step append (null new_k: none): row s of new_k/new_v ([num_seqs][num_kv_heads]
    // [head_dim], in_dtype) goes to slot new_slots[s], which lies in sequence s's last block
    const void* new_k;
    const void* new_v;
    const int64_t* new_slots;
    int in_dtype;
    // new tokens per sequence (tensor-core kernel; 0 or 1: one): the G query columns of a KV head
    // are q_len tokens x (num_heads / num_kv_heads) heads, token-major, causal within the chunk
    int q_len;
    // FP8 caches: one dequantisation scale per KV head ([num_kv_heads], device; null: the
    // per-tensor k_scale / v_scale_in)
    const float* k_head_scales;
    const float* v_head_scales;
    // failure-path test hook (tensor-core kernel): 1 + the unit whose stage the producer never
    // hands to its consumers, so their bounded wait runs out; 0 = none
    int withheld_unit;
    // Shared-prefix decode, suffix pass (null: none): sequence s starts at logical block
    // skip_blocks[s] of its table (the blocks before it are read by the prefix pass) and writes
    // fp32 partials instead of `out` whenever skip_blocks[s] > 0.
    const int32_t* skip_blocks;
    // Shared-prefix decode, prefix pass (null: none): the kernel's "sequences" are the plan's
    // groups (block_tables = group rows, seq_lens = their token counts, num_seqs = groups);
    // column c of KV head h of group gi is query head h * Gq + c % Gq of member c / Gq, i.e. of
    // sequence pfx_members[pfx_offsets[gi] + c / Gq], which sees pfx_shared[that sequence]
    // blocks of the row. Gq = num_heads / num_kv_heads.
    const int32_t* pfx_members;
    const int32_t* pfx_offsets;
    const int32_t* pfx_shared;
    // members a group may hold (host-checked: pfx_max_group * Gq <= 32); larger groups are flagged
    int pfx_max_group;
    int pfx_num_seqs;   // sequences of the batch (members must lie in [0, pfx_num_seqs))
    // 1: execute griddepcontrol.wait before the grid exits (a suffix pass launched behind the
    // prefix pass, so that the merge's wait covers both)
    int wait_prior_at_exit;
    // Tensor-core kernels: tail chunks per run (0: one static run per CTA) and the workspace
    // counter they are claimed from (zero before the launch; the merge kernel clears it after)
    int tail_chunks;
    int32_t* chunk_ctr;
    // the chunk schedule's thresholds: units per CTA below which the split stays static, and the
    // smallest tail chunk (kMinUnitsForTail / kMinTailChunk unless a kernel's units are larger)
    int tail_min_units;
    int tail_min_chunk;
    // partial slots the workspace holds (pieces of split streams, slot_floats floats each)
    long long partial_slots;
    // Per-chunk completion stamps (null: none): a CTA stores chunk_stamp(epoch) at
    // chunk_done[chunk] once the chunk's pieces are written, and the merge starts on a split stream
    // as soon as its chunks carry this call's stamp. epoch differs from call to call.
    unsigned long long* chunk_done;
    uint32_t epoch;
};

// The completion stamp of a chunk in the call with this epoch: the epoch and its complement, a
// pattern that no value the workspace held before (partials, stamps of other calls) can match.
__host__ __device__ __forceinline__ unsigned long long chunk_stamp(uint32_t epoch)
{
    return ((unsigned long long)epoch << 32) | (unsigned long long)(~epoch);
}

// One request to the warp-MMA kernels of a shape (decode_mma_dispatch.cuh).
struct MmaOp {
    enum Kind { kLaunch = 0, kOccupancy = 1, kLaunchSharedPrefix = 2, kPrefixOccupancy = 3 };
    int kind;
    const DecodeParams* p;    // the decode (or the shared-prefix suffix pass)
    const DecodeParams* pp;   // the shared-prefix prefix pass (kLaunchSharedPrefix)
    int nruns;                // runs of p
    int runs_p;               // runs of pp
    cudaStream_t stream;
    int* occ;                 // out: CTAs per SM (occupancy kinds)
};

// Kernel selection: warp-MMA kernel for bf16 / E4M3 caches of supported shapes,
// CUDA-core kernel otherwise. Returns PKV_ERR_SHAPE for unsupported shapes.
int decode_dispatch(int q_dtype, int kv_dtype, int head_dim, int block_size, int group,
                    const DecodeParams& p, int nruns, cudaStream_t stream, int* occupancy_out);
bool mma_supported(int kv_dtype, int head_dim, int block_size, int group, int num_kv_heads);
int mma_head_group(int kv_dtype, int head_dim, int block_size, int num_kv_heads);
int decode_mma_dispatch(int kv_dtype, int D, int BS, int G, int HG, const DecodeParams& p, int nruns,
                        cudaStream_t st, int* occ);
// Any MmaOp on the warp-MMA kernels of a cache type and shape.
int decode_mma_op(int kv_dtype, int D, int BS, int G, int HG, const MmaOp& op);

// The fused step's append + decode in one launch (warp-MMA kernel only).
bool step_fusable(int q_dtype, int kv_dtype, int head_dim, int block_size, int group, int num_kv_heads);

int cache_dispatch(const void* k, const void* v, void* k_cache, void* v_cache, const int64_t* slot_mapping,
                   int num_tokens, int num_kv_heads, int head_dim, int block_size, int num_blocks,
                   int in_dtype, int kv_dtype, float k_scale, float v_scale, const float* k_head_scales,
                   const float* v_head_scales, int32_t* err, cudaStream_t stream);

// Rows of the decode-step append (paged_decode_step): row s of k / v goes to slots[s].
struct AppendArgs {
    const void* k;
    const void* v;
    const int64_t* slots;
    int in_dtype;
};

// Host checks of a decode call (what paged_attention_decode validates before launching), the
// partition count and the kernels' parameters; queues nothing. Returns a pkv_status; on PKV_OK,
// *runs is the partition count to launch with, or 0 when there is nothing to launch.
int decode_prepare(void* out, const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                   const int32_t* seq_lens, int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                   int block_size, float scale, int max_blocks_per_seq, int num_blocks, int q_dtype, int kv_dtype,
                   float k_scale, float v_scale, int num_partitions, void* workspace, size_t workspace_bytes,
                   const AppendArgs* app, int withheld_unit, int q_len, const float* k_head_scales,
                   const float* v_head_scales, DecodeParams* p_out, int* runs);

// Raise a kernel's dynamic shared-memory limit to at least `bytes` on the current device (cached).
bool ensure_smem_attribute(const void* kernel, size_t bytes);

}  // namespace pkv
