// Decode-step KV append (reshape_and_cache) for sm_100a.
//
// Each decode step produces one new K row and one new V row per KV head and
// writes them into the paged cache ("vLLM inference cost optimisation",
// developer.aliyun.com, section 1: generate the new K/V and write them into
// the KV cache). Row t goes to slot slot_mapping[t]: physical block
// slot / block_size, offset slot % block_size; a negative slot is padding.
//
// Purely bandwidth-bound: one thread moves 8 elements of one (token, head,
// K-or-V) row with 16-byte (or 2x16-byte) loads and one store, consecutive
// threads cover consecutive 8-element pieces, so each row is read and written
// with full coalescing. For an E4M3 cache the fp32 value x / scale (IEEE
// division) is converted with the hardware round-to-nearest-even, saturating
// conversion (cuda_fp8.h), 8 codes per 8-byte store.
#include <cstdint>
#include <type_traits>

#include "device.cuh"

#include "pkv_internal.h"

namespace pkv {

namespace {

// TIN: float or bf16 input rows; TC: cache element (same as TIN, or uint8_t FP8 codes of format FMT).
template <class TIN, class TC, __nv_fp8_interpretation_t FMT = __NV_E4M3>
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(
    const TIN* __restrict__ k, const TIN* __restrict__ v, TC* __restrict__ kc, TC* __restrict__ vc,
    const int64_t* __restrict__ slots, int num_tokens, int num_kv_heads, int head_dim, int block_size,
    long long capacity, float k_scale, float v_scale, const float* __restrict__ k_head_scales,
    const float* __restrict__ v_head_scales, int32_t* err)
{
    const int pieces = head_dim / 8;                 // 8-element pieces per row
    const long long per_token = (long long)num_kv_heads * pieces;
    const long long total = 2ll * num_tokens * per_token;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const bool is_v = idx >= (long long)num_tokens * per_token;
        const long long r = is_v ? idx - (long long)num_tokens * per_token : idx;
        const int t = (int)(r / per_token);
        const int rem = (int)(r - (long long)t * per_token);
        const int h = rem / pieces, c = rem - h * pieces;
        const long long slot = __ldg(slots + t);
        if (slot < 0)
            continue;
        if (slot >= capacity) {
            if (err && c == 0 && !is_v)
                atomicOr(err, PKV_DEVERR_SLOT);
            continue;
        }
        const long long blk = slot / block_size, off = slot - blk * block_size;
        const TIN* src = (is_v ? v : k) + ((long long)t * num_kv_heads + h) * head_dim + c * 8;
        TC* dst = (is_v ? vc : kc) + ((blk * num_kv_heads + h) * block_size + off) * head_dim + c * 8;
        const float sc = is_v ? (v_head_scales ? __ldg(v_head_scales + h) : v_scale)
                              : (k_head_scales ? __ldg(k_head_scales + h) : k_scale);
        if constexpr (std::is_same<TC, int8_t>::value)
            quant8_i8(src, reinterpret_cast<uint8_t*>(dst), sc);
        else if constexpr (sizeof(TC) == 1)
            quant8<FMT>(src, reinterpret_cast<uint8_t*>(dst), sc);
        else
            copy8(src, dst);
    }
}

template <class TIN, class TC, __nv_fp8_interpretation_t FMT = __NV_E4M3>
int launch_cache(const void* k, const void* v, void* kc, void* vc, const int64_t* slots, int num_tokens,
                 int num_kv_heads, int head_dim, int block_size, int num_blocks, float k_scale, float v_scale,
                 const float* k_head_scales, const float* v_head_scales, int32_t* err, cudaStream_t stream)
{
    const long long items = 2ll * num_tokens * num_kv_heads * (head_dim / 8);
    long long blocks = (items + 255) / 256;
    if (blocks > 148ll * 16)
        blocks = 148ll * 16;
    if (blocks < 1)
        blocks = 1;
    reshape_and_cache_kernel<TIN, TC, FMT><<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const TIN*>(k), static_cast<const TIN*>(v), static_cast<TC*>(kc), static_cast<TC*>(vc), slots,
        num_tokens, num_kv_heads, head_dim, block_size, (long long)num_blocks * block_size, k_scale, v_scale,
        k_head_scales, v_head_scales, err);
    return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_LAUNCH;
}

}  // namespace

int cache_dispatch(const void* k, const void* v, void* k_cache, void* v_cache, const int64_t* slot_mapping,
                   int num_tokens, int num_kv_heads, int head_dim, int block_size, int num_blocks, int in_dtype,
                   int kv_dtype, float k_scale, float v_scale, const float* k_head_scales,
                   const float* v_head_scales, int32_t* err, cudaStream_t stream)
{
#define PKV_CACHE(TIN, TC, ...)                                                                               \
    return launch_cache<TIN, TC, ##__VA_ARGS__>(k, v, k_cache, v_cache, slot_mapping, num_tokens, num_kv_heads, \
                                                head_dim, block_size, num_blocks, k_scale, v_scale,            \
                                                k_head_scales, v_head_scales, err, stream)
    if (in_dtype == PKV_F32 && kv_dtype == PKV_F32)
        PKV_CACHE(float, float);
    if (in_dtype == PKV_BF16 && kv_dtype == PKV_BF16)
        PKV_CACHE(__nv_bfloat16, __nv_bfloat16);
    if (in_dtype == PKV_F32 && kv_dtype == PKV_FP8_E4M3)
        PKV_CACHE(float, uint8_t);
    if (in_dtype == PKV_BF16 && kv_dtype == PKV_FP8_E4M3)
        PKV_CACHE(__nv_bfloat16, uint8_t);
    if (in_dtype == PKV_F32 && kv_dtype == PKV_FP8_E5M2)
        PKV_CACHE(float, uint8_t, __NV_E5M2);
    if (in_dtype == PKV_BF16 && kv_dtype == PKV_FP8_E5M2)
        PKV_CACHE(__nv_bfloat16, uint8_t, __NV_E5M2);
    if (in_dtype == PKV_F32 && kv_dtype == PKV_INT8)
        PKV_CACHE(float, int8_t);
    if (in_dtype == PKV_BF16 && kv_dtype == PKV_INT8)
        PKV_CACHE(__nv_bfloat16, int8_t);
#undef PKV_CACHE
    return PKV_ERR_DTYPE;
}

}  // namespace pkv
