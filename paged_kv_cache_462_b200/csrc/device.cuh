// Device-side building blocks shared by the kernels of libpagedkv:
// mbarrier + bulk-copy (TMA, non-tensor) primitives written as inline PTX,
// bounded waits, and conversions of cache chunks to fp32.
#pragma once

#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

namespace pkv {

constexpr unsigned kFullMask = 0xffffffffu;

__device__ __forceinline__ uint32_t smem_addr(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Make mbarrier initialisation visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking test of the phase with the given parity (never suspends the thread).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase of `bar` with the given parity to complete, giving up
// after about one second (or 2^26 polls), so that a lost arrival can never
// hang the GPU. Returns false on timeout.
constexpr uint64_t kWaitLimitNs = 1000000000ull;
constexpr uint32_t kWaitLimitPolls = 1u << 26;

__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity)
{
    if (mbar_test_wait(bar, parity))   // the common case, a phase already complete: no suspension
        return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 0; i < kWaitLimitPolls; ++i) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((i & 63u) == 63u && global_ns() - t0 > kWaitLimitNs)
            return false;
    }
    return false;
}

// One bulk global->shared copy (no tensor map, no multicast) completing on `bar`.
// dst and src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// Order this thread's earlier generic-proxy shared-memory accesses before its
// later async-proxy (bulk copy) accesses.
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void named_barrier_sync(int id, int threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// prefix[] is a per-sequence exclusive prefix sum of work units; returns the s with
// prefix[s] <= x < prefix[s+1] (sequences without units are never returned).
__device__ __forceinline__ int find_seq(const int* prefix, int num_seqs, int x)
{
    int lo = 0, hi = num_seqs;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (prefix[mid] <= x)
            lo = mid;
        else
            hi = mid;
    }
    return lo;
}

__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ------------------------------------------------------------------ dtypes
// An E4M3 byte is widened to fp32 by moving its sign to bit 31 and its 7
// exponent+mantissa bits to bits 26..20. The fp32 word then holds the code's
// value times 2^-120 exactly (normal codes become normal fp32 numbers with the
// exponent field equal to the E4M3 exponent field; subnormal codes become fp32
// subnormals), so the 2^120 is folded into the per-tensor scales instead.
constexpr float kE4M3Unbias = 1.329227995784915872903807060280344576e36f;  // 2^120

struct KvF32 {
    using T = float;
    static constexpr bool kInt8 = false;
    static constexpr int kBytes = 4;
    static constexpr float kUnbias = 1.0f;
};
struct KvBF16 {
    using T = __nv_bfloat16;
    static constexpr bool kInt8 = false;
    static constexpr int kBytes = 2;
    static constexpr float kUnbias = 1.0f;
};
struct KvE4M3 {
    using T = uint8_t;
    static constexpr bool kInt8 = false;
    static constexpr int kBytes = 1;
    static constexpr float kUnbias = kE4M3Unbias;
    static constexpr __nv_fp8_interpretation_t kFmt = __NV_E4M3;
};
// OCP E5M2 codes (tensor-core kernel only: widened exactly to f16 there)
struct KvE5M2 {
    using T = uint8_t;
    static constexpr bool kInt8 = false;
    static constexpr int kBytes = 1;
    static constexpr __nv_fp8_interpretation_t kFmt = __NV_E5M2;
};
// symmetric INT8 codes (tensor-core kernel only: widened exactly to f16 there)
struct KvI8 {
    using T = uint8_t;
    static constexpr bool kInt8 = true;
    static constexpr int kBytes = 1;
    static constexpr __nv_fp8_interpretation_t kFmt = __NV_E4M3;   // unused for integers
};

__device__ __forceinline__ void widen_word(KvF32, uint32_t w, float* f) { f[0] = __uint_as_float(w); }

__device__ __forceinline__ void widen_word(KvBF16, uint32_t w, float* f)
{
    f[0] = __uint_as_float(w << 16);
    f[1] = __uint_as_float(w & 0xffff0000u);
}

__device__ __forceinline__ void widen_word(KvE4M3, uint32_t w, float* f)
{
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int32_t top = static_cast<int32_t>(__byte_perm(w, 0u, 0x0444u | (i << 12)));
        f[i] = __uint_as_float(static_cast<uint32_t>(top >> 4) & 0x87f00000u);
    }
}

// Load CHUNK bytes (4, 8 or 16) from shared memory and widen to fp32.
template <class KV, int CHUNK>
__device__ __forceinline__ void load_widen(const uint8_t* p, float* f)
{
    constexpr int kPerWord = 4 / KV::kBytes;
    if constexpr (CHUNK == 16) {
        const uint4 u = *reinterpret_cast<const uint4*>(p);
        widen_word(KV{}, u.x, f + 0 * kPerWord);
        widen_word(KV{}, u.y, f + 1 * kPerWord);
        widen_word(KV{}, u.z, f + 2 * kPerWord);
        widen_word(KV{}, u.w, f + 3 * kPerWord);
    } else if constexpr (CHUNK == 8) {
        const uint2 u = *reinterpret_cast<const uint2*>(p);
        widen_word(KV{}, u.x, f + 0 * kPerWord);
        widen_word(KV{}, u.y, f + 1 * kPerWord);
    } else {
        static_assert(CHUNK == 4, "chunk is 4, 8 or 16 bytes");
        widen_word(KV{}, *reinterpret_cast<const uint32_t*>(p), f);
    }
}

// Load CHUNK bytes of cache elements from shared memory as fp32 pairs
// (element 2i in .x, 2i+1 in .y), for the packed fp32x2 FMA.
__device__ __forceinline__ void widen_word2(KvBF16, uint32_t w, float2* f)
{
    f[0] = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

__device__ __forceinline__ void widen_word2(KvE4M3, uint32_t w, float2* f)
{
    float t[4];
    widen_word(KvE4M3{}, w, t);
    f[0] = make_float2(t[0], t[1]);
    f[1] = make_float2(t[2], t[3]);
}

template <class KV, int CHUNK>
__device__ __forceinline__ void load_widen2(const uint8_t* p, float2* f)
{
    if constexpr (KV::kBytes == 4) {
        static_assert(CHUNK == 16 || CHUNK == 8, "fp32 chunk");
        if constexpr (CHUNK == 16) {
            const float4 u = *reinterpret_cast<const float4*>(p);
            f[0] = make_float2(u.x, u.y);
            f[1] = make_float2(u.z, u.w);
        } else {
            f[0] = *reinterpret_cast<const float2*>(p);
        }
    } else {
        constexpr int kPairsPerWord = 2 / KV::kBytes;   // bf16: 1, e4m3: 2
        if constexpr (CHUNK == 16) {
            const uint4 u = *reinterpret_cast<const uint4*>(p);
            widen_word2(KV{}, u.x, f + 0 * kPairsPerWord);
            widen_word2(KV{}, u.y, f + 1 * kPairsPerWord);
            widen_word2(KV{}, u.z, f + 2 * kPairsPerWord);
            widen_word2(KV{}, u.w, f + 3 * kPairsPerWord);
        } else if constexpr (CHUNK == 8) {
            const uint2 u = *reinterpret_cast<const uint2*>(p);
            widen_word2(KV{}, u.x, f + 0 * kPairsPerWord);
            widen_word2(KV{}, u.y, f + 1 * kPairsPerWord);
        } else {
            static_assert(CHUNK == 4, "chunk is 4, 8 or 16 bytes");
            widen_word2(KV{}, *reinterpret_cast<const uint32_t*>(p), f);
        }
    }
}

// Load N consecutive q elements (8 or 16 bytes per vector) from global memory as fp32.
template <int N>
__device__ __forceinline__ void load_q(const float* p, float* f)
{
#pragma unroll
    for (int i = 0; i < N; i += 4) {
        const float4 u = __ldg(reinterpret_cast<const float4*>(p + i));
        f[i] = u.x; f[i + 1] = u.y; f[i + 2] = u.z; f[i + 3] = u.w;
    }
}

template <int N>
__device__ __forceinline__ void load_q(const __nv_bfloat16* p, float* f)
{
    if constexpr (N % 8 == 0) {
#pragma unroll
        for (int i = 0; i < N; i += 8) {
            const uint4 u = __ldg(reinterpret_cast<const uint4*>(p + i));
            widen_word(KvBF16{}, u.x, f + i);
            widen_word(KvBF16{}, u.y, f + i + 2);
            widen_word(KvBF16{}, u.z, f + i + 4);
            widen_word(KvBF16{}, u.w, f + i + 6);
        }
    } else {
        static_assert(N == 4, "q vector of 4 or a multiple of 8 elements");
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
        widen_word(KvBF16{}, u.x, f);
        widen_word(KvBF16{}, u.y, f + 2);
    }
}

// ---- one 8-element piece of a K/V row, as the decode-step append writes it ------------
__device__ __forceinline__ void load8(const float* p, float* f)
{
    const float4 a = *reinterpret_cast<const float4*>(p);
    const float4 b = *reinterpret_cast<const float4*>(p + 4);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* f)
{
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    widen_word(KvBF16{}, u.x, f + 0);
    widen_word(KvBF16{}, u.y, f + 2);
    widen_word(KvBF16{}, u.z, f + 4);
    widen_word(KvBF16{}, u.w, f + 6);
}

template <class T>
__device__ __forceinline__ void copy8(const T* src, T* dst)
{
    if constexpr (sizeof(T) == 4) {
        reinterpret_cast<float4*>(dst)[0] = reinterpret_cast<const float4*>(src)[0];
        reinterpret_cast<float4*>(dst)[1] = reinterpret_cast<const float4*>(src)[1];
    } else {
        *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
    }
}

// 8 values -> 8 codes of format FMT: x / scale (IEEE fp32 division), round to nearest even,
// saturated to the largest finite value
template <__nv_fp8_interpretation_t FMT = __NV_E4M3, class TIN>
__device__ __forceinline__ void quant8(const TIN* src, uint8_t* dst, float scale)
{
    float f[8];
    load8(src, f);
    uint32_t w[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t packed = 0;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const float2 y = make_float2(__fdiv_rn(f[4 * h + 2 * i], scale), __fdiv_rn(f[4 * h + 2 * i + 1], scale));
            const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(y, __NV_SATFINITE, FMT);
            packed |= static_cast<uint32_t>(c) << (16 * i);
        }
        w[h] = packed;
    }
    *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
}


// 8 values -> 8 symmetric INT8 codes: x / scale (IEEE fp32 division), nearest integer with ties
// to even, clamped to +-127; NaN -> 0
template <class TIN>
__device__ __forceinline__ void quant8_i8(const TIN* src, uint8_t* dst, float scale)
{
    float f[8];
    load8(src, f);
    uint32_t w[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t packed = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float y = __fdiv_rn(f[4 * h + i], scale);
            const int c = (y != y) ? 0 : __float2int_rn(fminf(fmaxf(y, -127.0f), 127.0f));
            packed |= (static_cast<uint32_t>(c) & 0xFFu) << (8 * i);
        }
        w[h] = packed;
    }
    *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
}

__device__ __forceinline__ float to_float(float x) { return x; }
__device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_float(float v, float* p) { *p = v; }
__device__ __forceinline__ void from_float(float v, __nv_bfloat16* p) { *p = __float2bfloat16_rn(v); }

}  // namespace pkv
