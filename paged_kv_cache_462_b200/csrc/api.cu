// C ABI of libpagedkv: argument validation, workspace layout and launch.
// Every entry point validates what the host can see and returns a pkv_status
// before launching anything; nothing here allocates, frees or synchronises
// (pkv_read_device_error excepted, which synchronises by design).
#include <atomic>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include <cuda.h>
#include <cuda_runtime.h>

#include "pkv_blocks.h"
#include "pkv_internal.h"

namespace pkv {

namespace {

std::mutex g_mu;
std::map<std::pair<const void*, int>, size_t> g_smem_set;   // (kernel, device) -> dynamic smem limit set
std::map<int, int> g_sm_count;                                // device -> SMs

int current_device()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return -1;
    return dev;
}

int sm_count(int dev)
{
    std::lock_guard<std::mutex> lock(g_mu);
    auto it = g_sm_count.find(dev);
    if (it != g_sm_count.end())
        return it->second;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    try {
        g_sm_count[dev] = n;
    } catch (...) {
    }
    return n;
}

bool group_supported(int g) { return g == 1 || g == 2 || g == 4 || g == 5 || g == 8; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int slot_floats_for(int group, int head_dim) { return (int)round_up((size_t)group * (head_dim + 2), 4); }

struct WorkspaceLayout {
    size_t counters_off, done_off, partials_off, bytes;
};

WorkspaceLayout layout_for(int num_seqs, int num_kv_heads, int group, int head_dim, long long runs)
{
    WorkspaceLayout w;
    const long long pairs = (long long)num_seqs * num_kv_heads;
    w.counters_off = kWorkspaceHeader;
    w.done_off = w.counters_off + round_up((size_t)pairs * 4, 256);
    // one completion stamp (8 bytes) per chunk
    w.partials_off = w.done_off + round_up((size_t)(runs * (1 + kTailChunksPerRun)) * 8, 256);
    // a chunk (a run's own or a tail chunk, 1 + kTailChunksPerRun per run at most) writes at most
    // one partial per (stream it touches, head of the stream's group)
    w.bytes = w.partials_off +
              (size_t)(runs * (1 + kTailChunksPerRun) * kMaxHeadGroup + pairs) * slot_floats_for(group, head_dim) * 4;
    return w;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A new value for every call (never 0, whose stamp a fresh zeroed workspace cannot hold anyway).
uint32_t next_epoch()
{
    static std::atomic<uint32_t> g_epoch{0};
    uint32_t e = g_epoch.fetch_add(1, std::memory_order_relaxed) + 1;
    if (e == 0)
        e = g_epoch.fetch_add(1, std::memory_order_relaxed) + 1;
    return e;
}

// 8-bit caches quantised with scales (FP8 formats and INT8)
bool is_fp8(int dtype) { return dtype == PKV_FP8_E4M3 || dtype == PKV_FP8_E5M2 || dtype == PKV_INT8; }

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!tried) {
        tried = true;
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

}  // namespace

bool make_cache_tensormap(CUtensorMap* map, const void* base, int kv_dtype, int head_dim, long long rows,
                          int box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    const int elt = kv_dtype == PKV_BF16 ? 2 : 1;
    const cuuint64_t dims[2] = {(cuuint64_t)head_dim, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)head_dim * elt};
    const cuuint32_t box[2] = {(cuuint32_t)(128 / elt), (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(map, kv_dtype == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                          const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool ensure_smem_attribute(const void* kernel, size_t bytes)
{
    const int dev = current_device();
    if (dev < 0)
        return false;
    std::lock_guard<std::mutex> lock(g_mu);
    auto key = std::make_pair(kernel, dev);
    auto it = g_smem_set.find(key);
    if (it != g_smem_set.end() && it->second >= bytes)
        return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
        return false;
    try {   // only a cache of the attribute: a failed insert just means it is set again next time
        g_smem_set[key] = bytes;
    } catch (...) {
    }
    return true;
}

// Host checks, partition count and launch parameters of a decode call; nothing is queued. On
// PKV_OK, *runs = 0 means there is nothing to launch (no sequences).
int decode_prepare(void* out, const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                   const int32_t* seq_lens, int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                   int block_size, float scale, int max_blocks_per_seq, int num_blocks, int q_dtype, int kv_dtype,
                   float k_scale, float v_scale, int num_partitions, void* workspace, size_t workspace_bytes,
                   const AppendArgs* app, int withheld_unit, int q_len, const float* k_head_scales,
                   const float* v_head_scales, DecodeParams* p_out, int* runs_out)
{
    *runs_out = 0;
    if (num_seqs < 0 || num_seqs > kMaxSeqs || num_heads <= 0 || num_kv_heads <= 0 ||
        num_heads % num_kv_heads != 0 || num_partitions < 0 || q_len < 1 || q_len > 8)
        return PKV_ERR_SHAPE;
    // query columns per KV head: q_len new tokens x the GQA group (the kernels' "group")
    const int group = num_heads / num_kv_heads * q_len;
    if (!group_supported(group) || (head_dim != 64 && head_dim != 128) ||
        (block_size != 8 && block_size != 16 && block_size != 32))
        return PKV_ERR_SHAPE;
    if (q_len > 1 && (app || !(q_dtype == PKV_BF16 && mma_supported(kv_dtype, head_dim, block_size, group,
                                                                       num_kv_heads))))
        return PKV_ERR_SHAPE;   // several new tokens: tensor-core kernel only, no fused append
    if ((k_head_scales || v_head_scales) &&
        (!k_head_scales || !v_head_scales || !is_fp8(kv_dtype) ||
         !(q_dtype == PKV_BF16 && mma_supported(kv_dtype, head_dim, block_size, group, num_kv_heads))))
        return PKV_ERR_SHAPE;   // per-head scales: both arrays, FP8 caches, tensor-core kernel
    if (!((q_dtype == PKV_F32 && kv_dtype == PKV_F32) || (q_dtype == PKV_BF16 && kv_dtype == PKV_BF16) ||
          (q_dtype == PKV_BF16 && is_fp8(kv_dtype))))
        return PKV_ERR_DTYPE;
    if (num_seqs == 0)
        return PKV_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens)
        return PKV_ERR_NULL;
    if (!workspace)
        return PKV_ERR_WORKSPACE;
    if (max_blocks_per_seq <= 0 || num_blocks <= 0)
        return PKV_ERR_SHAPE;
    if ((long long)num_seqs * max_blocks_per_seq * num_kv_heads >= (1ll << 31) ||
        (long long)max_blocks_per_seq * block_size >= (1ll << 31) ||
        (long long)num_blocks * num_kv_heads * block_size >= (1ll << 31))
        return PKV_ERR_SHAPE;
    if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(workspace))
        return PKV_ERR_SHAPE;

    int runs = num_partitions;
    if (runs == 0) {
        const int dev = current_device();
        const int sms = dev >= 0 ? sm_count(dev) : 0;
        if (sms <= 0)
            return PKV_ERR_DEVICE;
        DecodeParams probe;
        std::memset(&probe, 0, sizeof probe);
        probe.num_seqs = num_seqs;
        probe.num_kv_heads = num_kv_heads;
        int occ = 0;
        const int st = decode_dispatch(q_dtype, kv_dtype, head_dim, block_size, group, probe, 0, nullptr, &occ);
        if (st != PKV_OK)
            return st;
        if (occ < 1)
            return PKV_ERR_SHAPE;
        runs = sms * (occ > kMaxRunsPerSM ? kMaxRunsPerSM : occ);
    }
    const WorkspaceLayout lay = layout_for(num_seqs, num_kv_heads, group, head_dim, runs);
    if (workspace_bytes < lay.bytes)
        return PKV_ERR_WORKSPACE;

    const bool fp8 = is_fp8(kv_dtype);
    DecodeParams& p = *p_out;
    std::memset(&p, 0, sizeof p);
    p.out = out;
    p.q = q;
    p.k_cache = static_cast<const uint8_t*>(k_cache);
    p.v_cache = static_cast<const uint8_t*>(v_cache);
    p.block_tables = block_tables;
    p.seq_lens = seq_lens;
    p.num_seqs = num_seqs;
    p.num_heads = num_heads;
    p.num_kv_heads = num_kv_heads;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_blocks = num_blocks;
    p.scale = scale;
    p.k_scale = fp8 ? k_scale : 1.0f;
    p.v_scale_in = fp8 ? v_scale : 1.0f;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    p.err = reinterpret_cast<int32_t*>(ws);
    p.counters = reinterpret_cast<int32_t*>(ws + lay.counters_off);
    p.partials = reinterpret_cast<float*>(ws + lay.partials_off);
    p.slot_floats = slot_floats_for(group, head_dim);
    p.partial_slots = (long long)((workspace_bytes - lay.partials_off) / ((size_t)p.slot_floats * 4));
    p.chunk_done = reinterpret_cast<unsigned long long*>(ws + lay.done_off);
    p.epoch = next_epoch();
    p.q_len = q_len;
    p.k_head_scales = k_head_scales;
    p.v_head_scales = v_head_scales;
    p.tail_chunks = kTailChunksPerRun;
    p.tail_min_units = kMinUnitsForTail;
    p.tail_min_chunk = kMinTailChunk;
    p.chunk_ctr = reinterpret_cast<int32_t*>(ws) + 1;   // header word 1
    if (withheld_unit >= 0) {
        if (!(q_dtype == PKV_BF16 && mma_supported(kv_dtype, head_dim, block_size, group, num_kv_heads)))
            return PKV_ERR_SHAPE;   // the hook lives in the tensor-core kernel only
        p.withheld_unit = withheld_unit + 1;
    }
    if (app) {
        p.new_k = app->k;
        p.new_v = app->v;
        p.new_slots = app->slots;
        p.in_dtype = app->in_dtype;
    }
    *runs_out = runs;
    return PKV_OK;
}

}  // namespace pkv

using namespace pkv;

extern "C" {

const char* pkv_status_string(int status)
{
    switch (status) {
    case PKV_OK:
        return "ok";
    case PKV_ERR_NULL:
        return "a required pointer is NULL";
    case PKV_ERR_SHAPE:
        return "unsupported or inconsistent size, or a misaligned cache/row pointer";
    case PKV_ERR_DTYPE:
        return "unsupported dtype or dtype pair";
    case PKV_ERR_WORKSPACE:
        return "workspace missing or too small";
    case PKV_ERR_LAUNCH:
        return "kernel launch failed";
    case PKV_ERR_DEVICE:
        return "CUDA device query failed";
    case PKV_BM_NO_BLOCKS:
        return "block pool has no free block";
    case PKV_BM_UNKNOWN_SEQ:
        return "unknown sequence id";
    case PKV_BM_DUPLICATE_SEQ:
        return "sequence id already present";
    case PKV_BM_TABLE_FULL:
        return "sequence would exceed max_blocks_per_seq";
    default:
        return "unknown status";
    }
}

size_t paged_attention_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                      int num_partitions)
{
    if (num_seqs < 0 || num_kv_heads <= 0 || num_heads <= 0 || num_heads % num_kv_heads != 0)
        return 0;
    const int group = num_heads / num_kv_heads;
    if (!group_supported(group) || (head_dim != 64 && head_dim != 128) || num_partitions < 0)
        return 0;
    long long runs = num_partitions;
    if (runs == 0) {
        const int dev = current_device();
        const int sms = dev >= 0 ? sm_count(dev) : 0;
        if (sms <= 0)
            return 0;
        runs = (long long)sms * kMaxRunsPerSM;
    }
    return layout_for(num_seqs, num_kv_heads, group, head_dim, runs).bytes;
}

int pkv_workspace_init(void* workspace, size_t workspace_bytes, void* stream)
{
    if (!workspace)
        return PKV_ERR_NULL;
    if (workspace_bytes < kWorkspaceHeader)
        return PKV_ERR_WORKSPACE;
    return cudaMemsetAsync(workspace, 0, workspace_bytes, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? PKV_OK
               : PKV_ERR_LAUNCH;
}

int pkv_read_device_error(void* workspace, size_t workspace_bytes, int32_t* host_error, int clear, void* stream)
{
    if (!workspace || !host_error)
        return PKV_ERR_NULL;
    if (workspace_bytes < kWorkspaceHeader)
        return PKV_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t v = 0;
    if (cudaMemcpyAsync(&v, workspace, sizeof v, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return PKV_ERR_LAUNCH;
    if (cudaStreamSynchronize(st) != cudaSuccess)
        return PKV_ERR_LAUNCH;
    *host_error = v;
    if (clear && v != 0) {
        if (cudaMemsetAsync(workspace, 0, sizeof v, st) != cudaSuccess)
            return PKV_ERR_LAUNCH;
    }
    return PKV_OK;
}

int pkv_default_partitions(int head_dim, int block_size, int num_heads, int num_kv_heads, int kv_dtype)
{
    if (num_kv_heads <= 0 || num_heads % num_kv_heads != 0)
        return -PKV_ERR_SHAPE;
    const int dev = current_device();
    const int sms = dev >= 0 ? sm_count(dev) : 0;
    if (sms <= 0)
        return -PKV_ERR_DEVICE;
    const int q_dtype = kv_dtype == PKV_F32 ? PKV_F32 : PKV_BF16;
    DecodeParams p;
    std::memset(&p, 0, sizeof p);
    p.num_seqs = 1;
    p.num_kv_heads = num_kv_heads;
    int occ = 0;
    const int st = decode_dispatch(q_dtype, kv_dtype, head_dim, block_size, num_heads / num_kv_heads, p, 0,
                                   nullptr, &occ);
    if (st != PKV_OK)
        return -st;
    if (occ < 1)
        occ = 1;
    if (occ > kMaxRunsPerSM)
        occ = kMaxRunsPerSM;
    return sms * occ;
}

}  // extern "C"

namespace {

int decode_impl(void* out, const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                const int32_t* seq_lens, int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                float scale, int max_blocks_per_seq, int num_blocks, int q_dtype, int kv_dtype, float k_scale,
                float v_scale, int num_partitions, void* workspace, size_t workspace_bytes, void* stream,
                const AppendArgs* app, int withheld_unit = -1, int q_len = 1, const float* k_head_scales = nullptr,
                const float* v_head_scales = nullptr)
{
    DecodeParams p;
    int runs = 0;
    const int st = decode_prepare(out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, num_heads, num_kv_heads,
                                  head_dim, block_size, scale, max_blocks_per_seq, num_blocks, q_dtype, kv_dtype,
                                  k_scale, v_scale, num_partitions, workspace, workspace_bytes, app, withheld_unit,
                                  q_len, k_head_scales, v_head_scales, &p, &runs);
    if (st != PKV_OK || runs == 0)
        return st;
    return decode_dispatch(q_dtype, kv_dtype, head_dim, block_size, num_heads / num_kv_heads * q_len, p, runs,
                           static_cast<cudaStream_t>(stream), nullptr);
}

}  // namespace

extern "C" {

int paged_attention_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, const int32_t* seq_lens, int num_seqs, int num_heads,
                           int num_kv_heads, int head_dim, int block_size, float scale, int max_blocks_per_seq,
                           int num_blocks, int q_dtype, int kv_dtype, float k_scale, float v_scale,
                           int num_partitions, void* workspace, size_t workspace_bytes, void* stream)
{
    return decode_impl(out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, num_heads, num_kv_heads, head_dim,
                       block_size, scale, max_blocks_per_seq, num_blocks, q_dtype, kv_dtype, k_scale, v_scale,
                       num_partitions, workspace, workspace_bytes, stream, nullptr);
}

int paged_attention_decode_head_scales(void* out, const void* q, const void* k_cache, const void* v_cache,
                                       const int32_t* block_tables, const int32_t* seq_lens, int num_seqs,
                                       int num_heads, int num_kv_heads, int head_dim, int block_size, float scale,
                                       int max_blocks_per_seq, int num_blocks, int q_dtype, int kv_dtype,
                                       const float* k_head_scales, const float* v_head_scales, int num_partitions,
                                       void* workspace, size_t workspace_bytes, void* stream)
{
    if (!k_head_scales || !v_head_scales)
        return PKV_ERR_NULL;
    return decode_impl(out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, num_heads, num_kv_heads, head_dim,
                       block_size, scale, max_blocks_per_seq, num_blocks, q_dtype, kv_dtype, 1.0f, 1.0f,
                       num_partitions, workspace, workspace_bytes, stream, nullptr, -1, 1, k_head_scales,
                       v_head_scales);
}

int paged_attention_decode_mq(void* out, const void* q, const void* k_cache, const void* v_cache,
                              const int32_t* block_tables, const int32_t* seq_lens, int num_seqs, int q_len,
                              int num_heads, int num_kv_heads, int head_dim, int block_size, float scale,
                              int max_blocks_per_seq, int num_blocks, int q_dtype, int kv_dtype, float k_scale,
                              float v_scale, int num_partitions, void* workspace, size_t workspace_bytes,
                              void* stream)
{
    return decode_impl(out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, num_heads, num_kv_heads, head_dim,
                       block_size, scale, max_blocks_per_seq, num_blocks, q_dtype, kv_dtype, k_scale, v_scale,
                       num_partitions, workspace, workspace_bytes, stream, nullptr, -1, q_len);
}

int pkv_test_decode_timeout(void* out, const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_tables, const int32_t* seq_lens, int num_seqs, int num_heads,
                            int num_kv_heads, int head_dim, int block_size, float scale, int max_blocks_per_seq,
                            int num_blocks, int q_dtype, int kv_dtype, float k_scale, float v_scale,
                            int num_partitions, void* workspace, size_t workspace_bytes, int withheld_unit,
                            void* stream)
{
    if (withheld_unit < 0)
        return PKV_ERR_SHAPE;
    return decode_impl(out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, num_heads, num_kv_heads, head_dim,
                       block_size, scale, max_blocks_per_seq, num_blocks, q_dtype, kv_dtype, k_scale, v_scale,
                       num_partitions, workspace, workspace_bytes, stream, nullptr, withheld_unit);
}

int paged_decode_step(void* out, const void* q, void* k_cache, void* v_cache, const int32_t* block_tables,
                      const int32_t* seq_lens, int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                      int block_size, float scale, int max_blocks_per_seq, int num_blocks, int q_dtype, int kv_dtype,
                      float k_scale, float v_scale, int num_partitions, void* workspace, size_t workspace_bytes,
                      const void* new_k, const void* new_v, const int64_t* slot_mapping, int in_dtype, void* stream)
{
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0)
        return PKV_ERR_SHAPE;
    if (!((in_dtype == PKV_F32 || in_dtype == PKV_BF16) && (kv_dtype == in_dtype || is_fp8(kv_dtype))))
        return PKV_ERR_DTYPE;
    if (num_seqs == 0)
        return PKV_OK;
    if (!new_k || !new_v || !slot_mapping)
        return PKV_ERR_NULL;
    if (!workspace)
        return PKV_ERR_WORKSPACE;
    if (!aligned16(new_k) || !aligned16(new_v))
        return PKV_ERR_SHAPE;
    if (is_fp8(kv_dtype) && !(k_scale > 0.0f && v_scale > 0.0f))
        return PKV_ERR_SHAPE;
    const int group = num_heads / num_kv_heads;
    if (q_dtype == PKV_BF16 && mma_supported(kv_dtype, head_dim, block_size, group, num_kv_heads)) {
        const AppendArgs app{new_k, new_v, slot_mapping, in_dtype};
        return decode_impl(out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, num_heads, num_kv_heads,
                           head_dim, block_size, scale, max_blocks_per_seq, num_blocks, q_dtype, kv_dtype, k_scale,
                           v_scale, num_partitions, workspace, workspace_bytes, stream, &app);
    }
    // shapes the fused kernel does not cover: the two calls in stream order
    const int st = reshape_and_cache(new_k, new_v, k_cache, v_cache, slot_mapping, num_seqs, num_kv_heads, head_dim,
                                     block_size, num_blocks, in_dtype, kv_dtype, k_scale, v_scale,
                                     static_cast<int32_t*>(workspace), stream);
    if (st != PKV_OK)
        return st;
    return paged_attention_decode(out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, num_heads, num_kv_heads,
                                  head_dim, block_size, scale, max_blocks_per_seq, num_blocks, q_dtype, kv_dtype,
                                  k_scale, v_scale, num_partitions, workspace, workspace_bytes, stream);
}

}  // extern "C"

namespace {

// Bytes of the prefix pass's partials: a slot of 8 columns x (head_dim + 2) floats for every
// (run + stream) x column tile, streams = groups x KV heads.
size_t prefix_partials_bytes(int num_groups, int num_kv_heads, int head_dim, long long runs_p)
{
    if (num_groups <= 0)
        return 0;   // no prefix pass
    const size_t slot = round_up((size_t)8 * (head_dim + 2), 4) * 4;
    return (size_t)(runs_p * (1 + kTailChunksPerRun) + (long long)num_groups * num_kv_heads) * 4 * slot;
}

int shared_prefix_impl(void* out, const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* block_tables, const int32_t* seq_lens, int num_seqs, int num_heads,
                       int num_kv_heads, int head_dim, int block_size, float scale, int max_blocks_per_seq,
                       int num_blocks, int q_dtype, int kv_dtype, float k_scale, float v_scale,
                       const int32_t* group_members, const int32_t* group_offsets, const int32_t* group_tables,
                       const int32_t* group_lens, const int32_t* shared_blocks, int num_groups, int max_group,
                       int num_partitions, void* workspace, size_t workspace_bytes, const AppendArgs* app,
                       void* stream)
{
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0 ||
        num_groups < 0 || num_groups > num_seqs || max_group < 1)
        return PKV_ERR_SHAPE;
    const int Gq = num_heads / num_kv_heads;
    if (max_group * Gq > 32)
        return PKV_ERR_SHAPE;   // a group's queries of one KV head fill at most 4 column tiles of 8
    if (!(q_dtype == PKV_BF16 && mma_supported(kv_dtype, head_dim, block_size, Gq, num_kv_heads)))
        return q_dtype == PKV_BF16 && (kv_dtype == PKV_BF16 || is_fp8(kv_dtype)) ? PKV_ERR_SHAPE : PKV_ERR_DTYPE;
    if (num_seqs == 0)
        return PKV_OK;
    if (!shared_blocks || (num_groups > 0 && (!group_members || !group_offsets || !group_tables || !group_lens)))
        return PKV_ERR_NULL;
    DecodeParams ps;
    int runs_s = 0;
    int st = decode_prepare(out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, num_heads, num_kv_heads,
                            head_dim, block_size, scale, max_blocks_per_seq, num_blocks, q_dtype, kv_dtype, k_scale,
                            v_scale, num_partitions, workspace, workspace_bytes, app, -1, 1, nullptr, nullptr, &ps,
                            &runs_s);
    if (st != PKV_OK || runs_s == 0)
        return st;
    ps.skip_blocks = shared_blocks;

    int runs_p = num_partitions;
    const int HG = mma_head_group(kv_dtype, head_dim, block_size, num_kv_heads);
    if (runs_p == 0) {
        const int dev = current_device();
        const int sms = dev >= 0 ? sm_count(dev) : 0;
        if (sms <= 0)
            return PKV_ERR_DEVICE;
        DecodeParams probe;
        std::memset(&probe, 0, sizeof probe);
        probe.num_seqs = num_groups;
        probe.num_kv_heads = num_kv_heads;
        int occ = 0;
        MmaOp op{};
        op.kind = MmaOp::kPrefixOccupancy;
        op.p = &probe;
        op.occ = &occ;
        st = decode_mma_op(kv_dtype, head_dim, block_size, Gq, HG, op);
        if (st != PKV_OK)
            return st;
        if (occ < 1)
            return PKV_ERR_SHAPE;
        runs_p = sms * (occ > kMaxRunsPerSM ? kMaxRunsPerSM : occ);
    }
    const size_t suffix_bytes = layout_for(num_seqs, num_kv_heads, Gq, head_dim, runs_s).bytes;
    const size_t prefix_off = round_up(suffix_bytes, 256);
    if (workspace_bytes < prefix_off + prefix_partials_bytes(num_groups, num_kv_heads, head_dim, runs_p))
        return PKV_ERR_WORKSPACE;

    ps.chunk_done = nullptr;   // the shared-prefix merge waits for both passes' grids instead
    DecodeParams pp = ps;
    pp.num_seqs = num_groups;
    pp.seq_lens = group_lens;
    pp.block_tables = group_tables;
    pp.skip_blocks = nullptr;
    pp.new_k = pp.new_v = nullptr;
    pp.new_slots = nullptr;
    pp.partials = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + prefix_off);
    pp.slot_floats = (int)round_up((size_t)8 * (head_dim + 2), 4);
    pp.pfx_members = group_members;
    pp.pfx_offsets = group_offsets;
    pp.pfx_shared = shared_blocks;
    pp.pfx_max_group = max_group;
    pp.pfx_num_seqs = num_seqs;
    pp.chunk_ctr = reinterpret_cast<int32_t*>(workspace) + 2;   // header word 2: the prefix pass's claims

    MmaOp op{};
    op.kind = MmaOp::kLaunchSharedPrefix;
    op.p = &ps;
    op.pp = &pp;
    op.nruns = runs_s;
    op.runs_p = runs_p;
    op.stream = static_cast<cudaStream_t>(stream);
    return decode_mma_op(kv_dtype, head_dim, block_size, Gq, HG, op);
}

}  // namespace

extern "C" {

size_t paged_attention_shared_prefix_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                                    int num_groups, int num_partitions)
{
    const size_t base = paged_attention_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, num_partitions);
    if (base == 0 || num_groups < 0)
        return 0;
    long long runs = num_partitions;
    if (runs == 0) {
        const int dev = current_device();
        const int sms = dev >= 0 ? sm_count(dev) : 0;
        if (sms <= 0)
            return 0;
        runs = (long long)sms * kMaxRunsPerSM;
    }
    return round_up(base, 256) + prefix_partials_bytes(num_groups, num_kv_heads, head_dim, runs);
}

int paged_attention_decode_shared_prefix(void* out, const void* q, const void* k_cache, const void* v_cache,
                                         const int32_t* block_tables, const int32_t* seq_lens, int num_seqs,
                                         int num_heads, int num_kv_heads, int head_dim, int block_size, float scale,
                                         int max_blocks_per_seq, int num_blocks, int q_dtype, int kv_dtype,
                                         float k_scale, float v_scale, const int32_t* group_members,
                                         const int32_t* group_offsets, const int32_t* group_tables,
                                         const int32_t* group_lens, const int32_t* shared_blocks, int num_groups,
                                         int max_group, int num_partitions, void* workspace, size_t workspace_bytes,
                                         void* stream)
{
    return shared_prefix_impl(out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, num_heads, num_kv_heads,
                              head_dim, block_size, scale, max_blocks_per_seq, num_blocks, q_dtype, kv_dtype, k_scale,
                              v_scale, group_members, group_offsets, group_tables, group_lens, shared_blocks,
                              num_groups, max_group, num_partitions, workspace, workspace_bytes, nullptr, stream);
}

int paged_decode_step_shared_prefix(void* out, const void* q, void* k_cache, void* v_cache,
                                    const int32_t* block_tables, const int32_t* seq_lens, int num_seqs, int num_heads,
                                    int num_kv_heads, int head_dim, int block_size, float scale,
                                    int max_blocks_per_seq, int num_blocks, int q_dtype, int kv_dtype, float k_scale,
                                    float v_scale, const int32_t* group_members, const int32_t* group_offsets,
                                    const int32_t* group_tables, const int32_t* group_lens,
                                    const int32_t* shared_blocks, int num_groups, int max_group, int num_partitions,
                                    void* workspace, size_t workspace_bytes, const void* new_k, const void* new_v,
                                    const int64_t* slot_mapping, int in_dtype, void* stream)
{
    if (!((in_dtype == PKV_F32 || in_dtype == PKV_BF16) && (kv_dtype == in_dtype || is_fp8(kv_dtype))))
        return PKV_ERR_DTYPE;
    if (num_seqs > 0 && (!new_k || !new_v || !slot_mapping))
        return PKV_ERR_NULL;
    if (num_seqs > 0 && (!aligned16(new_k) || !aligned16(new_v)))
        return PKV_ERR_SHAPE;
    if (is_fp8(kv_dtype) && !(k_scale > 0.0f && v_scale > 0.0f))
        return PKV_ERR_SHAPE;
    const AppendArgs app{new_k, new_v, slot_mapping, in_dtype};
    return shared_prefix_impl(out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, num_heads, num_kv_heads,
                              head_dim, block_size, scale, max_blocks_per_seq, num_blocks, q_dtype, kv_dtype, k_scale,
                              v_scale, group_members, group_offsets, group_tables, group_lens, shared_blocks,
                              num_groups, max_group, num_partitions, workspace, workspace_bytes, &app, stream);
}

}  // extern "C"

namespace {

int cache_impl(const void* k, const void* v, void* k_cache, void* v_cache, const int64_t* slot_mapping,
               int num_tokens, int num_kv_heads, int head_dim, int block_size, int num_blocks, int in_dtype,
               int kv_dtype, float k_scale, float v_scale, const float* k_head_scales, const float* v_head_scales,
               int32_t* device_error, void* stream)
{
    if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0 || (head_dim != 64 && head_dim != 128) ||
        (block_size != 8 && block_size != 16 && block_size != 32))
        return PKV_ERR_SHAPE;
    if (!((in_dtype == PKV_F32 || in_dtype == PKV_BF16) &&
          (kv_dtype == in_dtype || is_fp8(kv_dtype))))
        return PKV_ERR_DTYPE;
    if (num_tokens == 0)
        return PKV_OK;
    if (!k || !v || !k_cache || !v_cache || !slot_mapping)
        return PKV_ERR_NULL;
    if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache))
        return PKV_ERR_SHAPE;
    if (is_fp8(kv_dtype) && !k_head_scales && !(k_scale > 0.0f && v_scale > 0.0f))
        return PKV_ERR_SHAPE;
    return cache_dispatch(k, v, k_cache, v_cache, slot_mapping, num_tokens, num_kv_heads, head_dim, block_size,
                          num_blocks, in_dtype, kv_dtype, k_scale, v_scale, k_head_scales, v_head_scales,
                          device_error, static_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" {

int reshape_and_cache(const void* k, const void* v, void* k_cache, void* v_cache, const int64_t* slot_mapping,
                      int num_tokens, int num_kv_heads, int head_dim, int block_size, int num_blocks, int in_dtype,
                      int kv_dtype, float k_scale, float v_scale, int32_t* device_error, void* stream)
{
    return cache_impl(k, v, k_cache, v_cache, slot_mapping, num_tokens, num_kv_heads, head_dim, block_size,
                      num_blocks, in_dtype, kv_dtype, k_scale, v_scale, nullptr, nullptr, device_error, stream);
}

int reshape_and_cache_head_scales(const void* k, const void* v, void* k_cache, void* v_cache,
                                  const int64_t* slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                                  int block_size, int num_blocks, int in_dtype, int kv_dtype,
                                  const float* k_head_scales, const float* v_head_scales, int32_t* device_error,
                                  void* stream)
{
    if (!is_fp8(kv_dtype))
        return PKV_ERR_DTYPE;
    if (num_tokens > 0 && (!k_head_scales || !v_head_scales))
        return PKV_ERR_NULL;
    return cache_impl(k, v, k_cache, v_cache, slot_mapping, num_tokens, num_kv_heads, head_dim, block_size,
                      num_blocks, in_dtype, kv_dtype, 1.0f, 1.0f, k_head_scales, v_head_scales, device_error,
                      stream);
}

}  // extern "C"
