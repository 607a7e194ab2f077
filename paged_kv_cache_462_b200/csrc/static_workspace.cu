// paged_attention_decode_static: the decode entry point for callers that cannot
// allocate device memory.
//
// Some callers have no way to obtain a workspace: code that runs while a CUDA
// graph is being captured (cudaMalloc is not allowed then), plug-ins and custom
// operators whose host framework owns every allocation and forbids allocating
// during execution, and embedded or real-time hosts that reserve all memory at
// start-up. This entry point takes the same inputs and outputs as
// paged_attention_decode but uses, as its scratch, one fixed array that lives in
// the library itself: every GPU that loads the library holds it until the
// process exits. Nothing here calls cudaMalloc, cudaFree or any allocating
// routine.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "pkv_internal.h"

namespace {

constexpr size_t kStaticWorkspaceBytes = 32u << 20;   // 32 MiB per GPU

// The scratch array. In host code its name is only a host-side stand-in, never a
// device address: the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_ws_addr[kMaxDevices] = {};

// Device address of the array on the current device (looked up once per device, with that
// device current; the lookup happens on the first call made on each device).
void* static_workspace(int dev)
{
    if (dev < 0 || dev >= kMaxDevices)
        return nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_ws_addr[dev] == nullptr) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_static_workspace) != cudaSuccess)
            return nullptr;
        g_ws_addr[dev] = ptr;
    }
    return g_ws_addr[dev];
}

}  // namespace

extern "C" PKV_API int paged_attention_decode_static(
    void* out, const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
    const int32_t* seq_lens, int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size, float scale,
    int max_blocks_per_seq, int num_blocks, int q_dtype, int kv_dtype, float k_scale, float v_scale,
    int num_partitions, void* stream)
{
    // reject what does not fit before touching the device
    const size_t need = paged_attention_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, num_partitions);
    if (need == 0)
        return PKV_ERR_SHAPE;
    if (need > kStaticWorkspaceBytes)
        return PKV_ERR_WORKSPACE;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return PKV_ERR_DEVICE;
    void* ws = static_workspace(dev);
    if (ws == nullptr)
        return PKV_ERR_DEVICE;
    // The array keeps whatever the previous call left. The error word and the per-(sequence,
    // KV head) arrival counters must start at zero: clear them (header + counters) first.
    const size_t pairs = (size_t)(num_seqs > 0 ? num_seqs : 0) * (size_t)(num_kv_heads > 0 ? num_kv_heads : 0);
    const size_t zero_bytes = pkv::kWorkspaceHeader + (pairs * 4 + 255) / 256 * 256;
    if (cudaMemsetAsync(ws, 0, zero_bytes < need ? zero_bytes : need, static_cast<cudaStream_t>(stream)) !=
        cudaSuccess)
        return PKV_ERR_LAUNCH;
    return paged_attention_decode(out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, num_heads, num_kv_heads,
                                  head_dim, block_size, scale, max_blocks_per_seq, num_blocks, q_dtype, kv_dtype,
                                  k_scale, v_scale, num_partitions, ws, kStaticWorkspaceBytes, stream);
}
