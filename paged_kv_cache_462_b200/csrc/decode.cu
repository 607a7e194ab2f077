// Dispatch of paged_attention_decode: the tcgen05 kernel (decode_tc05.cuh) for E4M3 / E5M2
// caches with head_dim 128, block size 16 or 32 and a multiple of 128 / block size KV heads; the
// warp-MMA kernel (decode_mma.cuh) for bf16 and INT8 caches and the other E4M3 / E5M2 shapes it
// covers (and the shared-prefix passes of every 8-bit and bf16 cache); the CUDA-core kernel
// (decode_kernel.cuh) for fp32 caches and the other bf16 / E4M3 shapes (E5M2 has no CUDA-core
// form).
#include <atomic>

#include "decode_kernel.cuh"

namespace pkv {

int decode_dispatch_f32(int D, int BS, int G, const DecodeParams& p, int nruns, cudaStream_t st, int* occ);
int decode_dispatch_bf16(int D, int BS, int G, const DecodeParams& p, int nruns, cudaStream_t st, int* occ);
int decode_dispatch_e4m3(int D, int BS, int G, const DecodeParams& p, int nruns, cudaStream_t st, int* occ);
int decode_mma_dispatch_bf16(int D, int BS, int G, int HG, const MmaOp& op);
int decode_mma_dispatch_e4m3(int D, int BS, int G, int HG, const MmaOp& op);
int decode_mma_dispatch_e5m2(int D, int BS, int G, int HG, const MmaOp& op);
int decode_mma_dispatch_i8(int D, int BS, int G, int HG, const MmaOp& op);

int decode_mma_op(int kv_dtype, int D, int BS, int G, int HG, const MmaOp& op)
{
    if (kv_dtype == PKV_BF16)
        return decode_mma_dispatch_bf16(D, BS, G, HG, op);
    if (kv_dtype == PKV_FP8_E4M3)
        return decode_mma_dispatch_e4m3(D, BS, G, HG, op);
    if (kv_dtype == PKV_FP8_E5M2)
        return decode_mma_dispatch_e5m2(D, BS, G, HG, op);
    if (kv_dtype == PKV_INT8)
        return decode_mma_dispatch_i8(D, BS, G, HG, op);
    return PKV_ERR_DTYPE;
}

int decode_mma_dispatch(int kv_dtype, int D, int BS, int G, int HG, const DecodeParams& p, int nruns,
                        cudaStream_t st, int* occ)
{
    MmaOp op{};
    op.kind = occ ? MmaOp::kOccupancy : MmaOp::kLaunch;
    op.p = &p;
    op.nruns = nruns;
    op.stream = st;
    op.occ = occ;
    return decode_mma_op(kv_dtype, D, BS, G, HG, op);
}

bool mma_supported(int kv_dtype, int head_dim, int block_size, int group, int num_kv_heads)
{
    if (kv_dtype != PKV_BF16 && kv_dtype != PKV_FP8_E4M3 && kv_dtype != PKV_FP8_E5M2 && kv_dtype != PKV_INT8)
        return false;
    if (block_size != 16 && block_size != 32)
        return false;
    if (group > 8)
        return false;
    if (kv_dtype == PKV_BF16 ? (head_dim != 64 && head_dim != 128) : head_dim != 128)
        return false;
    return mma_head_group(kv_dtype, head_dim, block_size, num_kv_heads) > 0;
}

bool step_fusable(int q_dtype, int kv_dtype, int head_dim, int block_size, int group, int num_kv_heads)
{
    return q_dtype == PKV_BF16 && mma_supported(kv_dtype, head_dim, block_size, group, num_kv_heads);
}

// Largest head group in {4, 2, 1} that divides num_kv_heads and keeps a stage (K + V) within
// 32 KB: two CTAs (two independent copy pipelines) per SM, 5 warps each.
int mma_head_group(int kv_dtype, int head_dim, int block_size, int num_kv_heads)
{
    const int elt = kv_dtype == PKV_BF16 ? 2 : 1;
    for (int hg = 4; hg >= 1; hg /= 2) {
        if (num_kv_heads % hg != 0)
            continue;
        if (2ll * hg * block_size * head_dim * elt <= 32 * 1024)
            return hg;
    }
    return 0;
}

int decode_tc05_dispatch(int kv_dtype, int D, int BS, int G, const DecodeParams& p, int nruns, cudaStream_t st,
                         int* occ);

// the tcgen05 kernel's unit is one block of 128 / block_size KV heads
bool tc05_supported(int q_dtype, int kv_dtype, int head_dim, int block_size, int group, int num_kv_heads)
{
    return q_dtype == PKV_BF16 && (kv_dtype == PKV_FP8_E4M3 || kv_dtype == PKV_FP8_E5M2) && head_dim == 128 &&
           (block_size == 16 || block_size == 32) && num_kv_heads % (128 / block_size) == 0 &&
           (group == 1 || group == 2 || group == 4 || group == 5 || group == 8);
}

std::atomic<int> g_fp8_kernel{PKV_FP8_KERNEL_MMA};

int decode_dispatch(int q_dtype, int kv_dtype, int D, int BS, int G, const DecodeParams& p, int nruns,
                    cudaStream_t st, int* occupancy_out)
{
    // FP8 caches on the tcgen05 kernel (8-bit products on the fifth-generation tensor cores)
    // when it is chosen and covers the shape
    if (g_fp8_kernel.load(std::memory_order_relaxed) == PKV_FP8_KERNEL_TCGEN05 &&
        tc05_supported(q_dtype, kv_dtype, D, BS, G, p.num_kv_heads))
        return decode_tc05_dispatch(kv_dtype, D, BS, G, p, nruns, st, occupancy_out);
    if (q_dtype == PKV_BF16 && mma_supported(kv_dtype, D, BS, G, p.num_kv_heads))
        return decode_mma_dispatch(kv_dtype, D, BS, G, mma_head_group(kv_dtype, D, BS, p.num_kv_heads), p, nruns,
                                   st, occupancy_out);
    if (q_dtype == PKV_F32 && kv_dtype == PKV_F32)
        return decode_dispatch_f32(D, BS, G, p, nruns, st, occupancy_out);
    if (q_dtype == PKV_BF16 && kv_dtype == PKV_BF16)
        return decode_dispatch_bf16(D, BS, G, p, nruns, st, occupancy_out);
    if (q_dtype == PKV_BF16 && kv_dtype == PKV_FP8_E4M3)
        return decode_dispatch_e4m3(D, BS, G, p, nruns, st, occupancy_out);
    return PKV_ERR_DTYPE;
}

}  // namespace pkv

extern "C" PKV_API int pkv_set_fp8_kernel(int which)
{
    if (which != PKV_FP8_KERNEL_MMA && which != PKV_FP8_KERNEL_TCGEN05)
        return -PKV_ERR_SHAPE;
    return pkv::g_fp8_kernel.exchange(which);
}
