// paged_attention_decode_static: the decode entry point for callers that cannot
// allocate device memory.
//
// Some callers have no way to obtain a workspace: plug-ins and custom operators
// whose host framework owns every allocation and forbids allocating while they
// run, embedded or real-time hosts that reserve all device memory at start-up,
// and latency-bound serving loops that cannot afford cudaMalloc's implicit
// device synchronisation. This entry point takes the same inputs and outputs as
// paged_attention_decode but uses, as its scratch, one fixed array that lives in
// the library itself: every GPU that loads the library holds it until the
// process exits. Nothing here calls cudaMalloc, cudaFree or any allocating
// routine.
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "pkv_internal.h"

namespace {

constexpr size_t kStaticWorkspaceBytes = 32u << 20;   // 32 MiB per GPU

// The scratch array. In host code its name is only a host-side stand-in, never a
// device address: the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

constexpr int kMaxDevices = 64;
std::mutex g_mu;
struct Cached {
    unsigned long long ctx_id;   // context the address belongs to (0: none yet)
    void* addr;
};
Cached g_ws[kMaxDevices] = {};

// Unique id of the calling thread's current context (ids are never reused within a process, so
// a context created again after cudaDeviceReset gets a new one); 0 if it cannot be read.
unsigned long long current_context_id()
{
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static bool tried = false;
    if (!tried) {   // under g_mu
        tried = true;
        void* p1 = nullptr;
        void* p2 = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p1, cudaEnableDefault, &q1) == cudaSuccess &&
            q1 == cudaDriverEntryPointSuccess &&
            cudaGetDriverEntryPoint("cuCtxGetId", &p2, cudaEnableDefault, &q2) == cudaSuccess &&
            q2 == cudaDriverEntryPointSuccess) {
            get_current = reinterpret_cast<CtxGetCurrentFn>(p1);
            get_id = reinterpret_cast<CtxGetIdFn>(p2);
        }
    }
    if (!get_current || !get_id)
        return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of the array in the current context of device `dev`, looked up with that
// device current the first time a context is seen (and again whenever the device's context
// changes, e.g. after cudaDeviceReset, when the module is loaded anew and the array may move).
void* static_workspace(int dev)
{
    if (dev < 0 || dev >= kMaxDevices)
        return nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    unsigned long long id = current_context_id();
    void* ptr = nullptr;
    if (id == 0) {   // no context current yet (first runtime use on this thread, or after a reset)
        if (cudaGetSymbolAddress(&ptr, g_static_workspace) != cudaSuccess)   // initialises it
            return nullptr;
        id = current_context_id();
        if (id == 0)
            return nullptr;
    }
    if (g_ws[dev].addr != nullptr && g_ws[dev].ctx_id == id)
        return g_ws[dev].addr;
    if (ptr == nullptr && cudaGetSymbolAddress(&ptr, g_static_workspace) != cudaSuccess)
        return nullptr;
    g_ws[dev] = Cached{id, ptr};
    return ptr;
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
    if (need > kStaticWorkspaceBytes)
        return PKV_ERR_WORKSPACE;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return PKV_ERR_DEVICE;
    void* ws = static_workspace(dev);
    if (ws == nullptr)
        return PKV_ERR_DEVICE;
    // every host check of paged_attention_decode, before anything is queued on `stream`
    pkv::DecodeParams p;
    int runs = 0;
    const int st = pkv::decode_prepare(out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, num_heads,
                                       num_kv_heads, head_dim, block_size, scale, max_blocks_per_seq, num_blocks,
                                       q_dtype, kv_dtype, k_scale, v_scale, num_partitions, ws,
                                       kStaticWorkspaceBytes, nullptr, -1, 1, nullptr, nullptr, &p, &runs);
    if (st != PKV_OK || runs == 0)
        return st;
    // The array keeps whatever the previous call left. The error word and the per-(sequence,
    // KV head) arrival counters must start at zero: clear them (header + counters) first.
    const size_t pairs = (size_t)num_seqs * (size_t)num_kv_heads;
    const size_t zero_bytes = pkv::kWorkspaceHeader + (pairs * 4 + 255) / 256 * 256;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, zero_bytes < need ? zero_bytes : need, s) != cudaSuccess)
        return PKV_ERR_LAUNCH;
    return pkv::decode_dispatch(q_dtype, kv_dtype, head_dim, block_size, num_heads / num_kv_heads, p, runs, s,
                                nullptr);
}
