// Paged decode attention for bf16 and 8-bit (E4M3, E5M2, INT8) caches on sm_100a: whole-block TMA
// tiles, one warp per KV head, warp-level tensor-core MMA with fp32 accumulation.
//
// Same result as the CUDA-core kernel (decode_kernel.cuh): for every sequence s
// and query head g, out[s][g] = softmax_t(scale * q . K_t) V_t over the
// seq_lens[s] cached tokens, K_t/V_t read through the block table
// ("vLLM inference cost optimisation", developer.aliyun.com, sections 2 and 4;
// wzjinhao.cn vLLM write-up, section 2.1), GQA head g -> KV head g / G.
//
// Why a second kernel: on the CUDA cores the q.K and p.V products of one
// 16-token tile cost ~900 (bf16) to ~1450 (E4M3, G = 5) warp instructions, so
// the decode step stayed issue-bound (measured with every tile resident in L2)
// well below the HBM rate. Here one tile costs ~100 instructions.
//
// Layout of the work:
//  * Unit = (sequence, head group of HG in {1, 2, 4} KV heads, logical block). The K
//    rows of a unit are HG*block_size consecutive rows of the pool
//    ([block][kv head][token][d]), i.e. one contiguous run (16 KB for bf16, 4
//    heads, block 16, d 128), fetched with 2-D TMA tensor copies whose 128-byte
//    swizzle makes the ldmatrix reads below bank-conflict free. Same for V.
//  * Units in (sequence, head group, block) order are cut into gridDim.x equal
//    runs (two or three CTAs per SM). Warp HG is the producer (block-table lookups, one
//    TMA copy per 128-byte-wide box, a ring of stages with full/empty
//    mbarriers); warps 0..HG-1 are consumers, warp w owning KV head
//    hg*HG + w of every unit, so a run's segment of one (sequence, head)
//    stream is finished by one warp without any CTA-wide barrier.
//  * Per 16-token tile: S^T = K Q^T with m16n8k16 MMA (16 tokens x 8 query
//    heads of the group, k = head_dim), scale, mask, online softmax with a lazy
//    running max (moved only when a tile max passes it by 8, in log2 units),
//    P^T re-laid out with 4 shuffles into the B operand of O^T += V^T P^T
//    (head_dim x 8 heads, k = 16 tokens). bf16 caches use bf16 MMA; 8-bit codes
//    are widened exactly to f16 (cvt.rn.f16x2.e4m3x2 / .e5m2x2 on a 16-bit half
//    of the loaded register; for INT8 a byte permute and one f16 subtraction)
//    and use f16 MMA, the per-tensor or per-head scales applied to the fp32
//    scores and outputs. For 8-bit caches the V codes come through the
//    transposed byte ldmatrix (four consecutive tokens of one d per lane) and
//    the tile's tokens take a fixed order (tok_of_row, v_tok) so that each
//    shuffled P^T word holds the two tokens of its MMA k pair.
//  * Split streams (a stream cut by a run boundary): each run's warp stores its
//    piece's fp32 partial (o, m, l) and moves on. A second, small kernel
//    launched as a programmatic dependent launch merges them (log-sum-exp, a
//    warp per stream and KV head). The streaming kernel only stamps each chunk
//    once its warps have written the chunk's pieces (a fence and one release
//    store per chunk), and a merge warp starts on a stream when the stream's
//    chunks carry this call's stamp: no atomic or merge sits in the streaming
//    kernel, whose memory system is saturated (a global round trip there costs
//    microseconds), and the result does not depend on timing.
#pragma once

#include <cstdint>
#include <type_traits>

#include <cuda.h>

#include "device.cuh"
#include "pkv_internal.h"

namespace pkv {

constexpr float kMmaRescaleSlack = 8.0f;  // log2 units
// INT8 caches: q.K on the integer tensor cores (true) or on f16 after widening the K codes (false)
constexpr bool kInt8Imma = true;
constexpr int kChunkRing = 16;             // chunk ids in flight between producer and consumers (> stages)

// ------------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// Two 16x16 byte matrices, transposed (sm_100a): lane i gives the address of row i & 15 of matrix
// i >> 4 (16 bytes); lane (g = lane >> 2, t = lane & 3) receives in r[2j] byte g and in r[2j + 1]
// byte g + 8 of rows 4t .. 4t + 3 of matrix j (row 4t + e in byte e).
__device__ __forceinline__ void ldsm_b8_x2_t(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m16n16.x2.trans.shared.b8 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

template <bool F16>
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    if constexpr (F16) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
            "{%0, %1, %2, %3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    } else {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
            "{%0, %1, %2, %3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
}

// D += A B with A 16x32 and B 32x8 of signed 8-bit integers, exact int32 sums
__device__ __forceinline__ void mma_16832_s8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Four values as signed 8-bit hi and lo codes of x = rint(v): hi = floor((x + 64) / 128), lo = x - 128 hi
// (hi + lo / 128 = x / 128 exactly; |x| < 8192 keeps hi in [-64, 64], lo in [-64, 63]). Byte i = value i.
__device__ __forceinline__ void split_s8x4(const float (&v)[4], uint32_t& hi, uint32_t& lo)
{
    hi = lo = 0u;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int x = __float2int_rn(v[i]);
        const int h = (x + 64) >> 7;
        hi |= (uint32_t)(h & 0xff) << (8 * i);
        lo |= (uint32_t)((x - (h << 7)) & 0xff) << (8 * i);
    }
}

// INT8 codes in bytes B0 and B1 of r as an exact f16x2 (byte B0 in the low half): the offset
// byte x + 128 as the mantissa of 1024.0 gives the f16 1152 + x; less 1152.
template <int B0, int B1>
__device__ __forceinline__ uint32_t widen2_i8(uint32_t r)
{
    const uint32_t x = __byte_perm(r ^ 0x80808080u, 0x64646464u, B0 | (4 << 4) | (B1 << 8) | (4 << 12));
    const __half2 h = __hsub2(*reinterpret_cast<const __half2*>(&x), __halves2half2(__ushort_as_half(0x6480),
                                                                                  __ushort_as_half(0x6480)));
    return *reinterpret_cast<const uint32_t*>(&h);
}

// The code pairs (bytes 0, 1) and (bytes 2, 3) of r widened exactly to f16x2 (the lower byte in
// the low half). E4M3 and E5M2: the hardware conversion of each 16-bit half of r, which takes no
// permute (every E5M2 value is an f16 value too; placing E4M3 bits in an f16 instead, the value
// times 2^-8, took more instructions and measured slower); INT8: widen2_i8.
template <class KV>
__device__ __forceinline__ void widen_halves(uint32_t r, uint32_t& w01, uint32_t& w23)
{
    if constexpr (!KV::kInt8 && KV::kFmt == __NV_E4M3) {
        asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
            "cvt.rn.f16x2.e4m3x2 %0, lo;\n\tcvt.rn.f16x2.e4m3x2 %1, hi;\n\t}"
            : "=r"(w01), "=r"(w23) : "r"(r));
    } else if constexpr (!KV::kInt8) {
        asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
            "cvt.rn.f16x2.e5m2x2 %0, lo;\n\tcvt.rn.f16x2.e5m2x2 %1, hi;\n\t}"
            : "=r"(w01), "=r"(w23) : "r"(r));
    } else {
        w01 = widen2_i8<0, 1>(r);
        w23 = widen2_i8<2, 3>(r);
    }
}

template <bool F16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi)
{
    if constexpr (F16) {
        const __half2 h = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<const uint32_t*>(&h);
    } else {
        const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<const uint32_t*>(&h);
    }
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Decode-step append fused into the producer warp: write the new token of sequence s (row s of
// new_k / new_v) for KV heads h0 .. h0+nh-1 into its slot, with the conversion reshape_and_cache
// uses, then order those writes before this warp's later TMA reads of the same block.
template <__nv_fp8_interpretation_t FMT, bool INT8, class TIN>
__device__ __forceinline__ void quant8_any(const TIN* src, uint8_t* dst, float scale)
{
    if constexpr (INT8)
        quant8_i8(src, dst, scale);
    else
        quant8<FMT>(src, dst, scale);
}

template <class TC, __nv_fp8_interpretation_t FMT = __NV_E4M3, bool INT8 = false>
__device__ __forceinline__ void append_rows(const DecodeParams& p, int s, int h0, int nh, int D, int BS, int lane,
                                            long long slot)
{
    const int pieces = D / 8;
    const long long blk = slot / BS, off = slot - blk * BS;
    TC* kc = reinterpret_cast<TC*>(const_cast<uint8_t*>(p.k_cache));
    TC* vc = reinterpret_cast<TC*>(const_cast<uint8_t*>(p.v_cache));
    for (int it = lane; it < 2 * nh * pieces; it += 32) {
        const bool is_v = it >= nh * pieces;
        const int r = is_v ? it - nh * pieces : it;
        const int h = h0 + r / pieces, c = r % pieces;
        const long long src_off = ((long long)s * p.num_kv_heads + h) * D + c * 8;
        TC* dst = (is_v ? vc : kc) + ((blk * p.num_kv_heads + h) * BS + off) * D + c * 8;
        const float sc = is_v ? (p.v_head_scales ? __ldg(p.v_head_scales + h) : p.v_scale_in)
                              : (p.k_head_scales ? __ldg(p.k_head_scales + h) : p.k_scale);
        if (p.in_dtype == PKV_F32) {
            const float* src = static_cast<const float*>(is_v ? p.new_v : p.new_k) + src_off;
            if constexpr (sizeof(TC) == 1)
                quant8_any<FMT, INT8>(src, reinterpret_cast<uint8_t*>(dst), sc);
        } else {
            const __nv_bfloat16* src = static_cast<const __nv_bfloat16*>(is_v ? p.new_v : p.new_k) + src_off;
            if constexpr (sizeof(TC) == 1)
                quant8_any<FMT, INT8>(src, reinterpret_cast<uint8_t*>(dst), sc);
            else
                copy8(src, reinterpret_cast<__nv_bfloat16*>(dst));
        }
    }
}

__device__ __forceinline__ void fence_proxy_async_global()
{
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// `last_phys`: physical block the sequence's last position maps to (-1 when its id was bad);
// a slot outside it is still written but flagged, since the decode may not see it
template <class KV>
__device__ __forceinline__ void append_new_token_impl(const DecodeParams& p, int s, int h0, int nh, int D, int BS,
                                                      int lane, int last_phys)
{
    const long long slot = __ldg(p.new_slots + s);
    if (slot >= 0) {
        if (lane == 0 && last_phys >= 0 && slot / BS != last_phys)
            atomicOr(p.err, PKV_DEVERR_SLOT);
        if (slot >= (long long)p.num_blocks * BS) {
            if (lane == 0)
                atomicOr(p.err, PKV_DEVERR_SLOT);
        } else if constexpr (KV::kBytes == 1) {
            append_rows<uint8_t, KV::kFmt, KV::kInt8>(p, s, h0, nh, D, BS, lane, slot);
        } else {
            append_rows<__nv_bfloat16>(p, s, h0, nh, D, BS, lane, slot);
        }
    }
    fence_proxy_async_global();
    __syncwarp();
}

// Row of `q` / `out` ([num_seqs][q_len][num_heads][d]) of query column c of KV head `head` of
// sequence s: column c is new token c / Gq of the sequence and query head head * Gq + c % Gq,
// Gq = num_heads / num_kv_heads (q_len = 1: column c is query head head * G + c).
__device__ __forceinline__ size_t query_row(const DecodeParams& p, int s, int head, int c)
{
    const int QL = p.q_len > 1 ? p.q_len : 1;
    const int Gq = p.num_heads / p.num_kv_heads;
    const int j = c / Gq, gh = c - j * Gq;
    return ((size_t)s * QL + j) * p.num_heads + (size_t)head * Gq + gh;
}

// ------------------------------------------------------------------ configuration

// PFX: the prefix pass of a shared-prefix decode. A unit is one KV head of one shared block of a
// group (HG = 1) and the kNT = 4 consumer warps take its 32 query columns (the group's members x
// their query heads), 8 each, against the same staged K/V tile.
template <class KV, int D, int BS, int G, int HG, bool PFX = false>
struct MmaCfg {
    // products: bf16 caches in bf16 MMA; 8-bit codes widened exactly to f16 (widen_halves) for f16 MMA,
    // q scaled per column by a power of two into f16's range; INT8 q.K on integer MMA (K codes as
    // they are, q as s8 hi + lo) when kInt8Imma
    static constexpr bool kF16 = KV::kBytes == 1;
    static constexpr bool kI8 = KV::kInt8 && kInt8Imma;
    static constexpr int kRowBytes = D * KV::kBytes;          // one token row of one head
    static constexpr int kBoxCols = 128 / KV::kBytes;         // elements per 128-byte box row
    static constexpr int kBoxes = kRowBytes / 128;            // boxes across head_dim
    static constexpr int kRows = HG * BS;                     // box rows: head-major, token-minor
    static constexpr int kBoxBytes = kRows * 128;
    static constexpr int kHalf = kBoxes * kBoxBytes;          // K (or V) part of a stage
    static constexpr int kStage = 2 * kHalf;
    static constexpr int kTT = BS / 16;                       // 16-token tiles per block
    static constexpr int kKS = D / 16;                        // q.K k-steps (16 d each)
    static constexpr int kDT = D / 16;                        // p.V m-tiles (16 d each)
    static constexpr int kNT = PFX ? 4 : 1;                   // column tiles (warps) per KV head
    static constexpr int W = HG * kNT;                        // consumer warps
    static constexpr int kThreads = (W + 1) * 32;
    // CTAs per SM: E4M3 tiles (16 KB stages) take three, for 12 consumer warps per SM to hide the
    // widening chain's latency; the same ~192 KB of stages per SM stay in flight either way
    static constexpr int kCtasPerSM = (KV::kBytes == 1 && kStage <= 16384) ? 3 : 2;
    static_assert(kRowBytes % 128 == 0, "rows are whole 128-byte swizzle spans");
    static_assert(BS % 16 == 0 && G <= 8 && HG <= 8, "tile shape");
    static_assert(kRows <= 256, "TMA box height");
    static_assert(KV::kBytes == 2 || D == 128, "8-bit MMA tiles: one 128-byte box across head_dim");
    static_assert(!PFX || (HG == 1 && G == 8), "prefix pass: one KV head per unit, 8 columns per warp");
};

// Byte offset of the 16-byte chunk `c` (0..7) of box row `r` in a 128B-swizzled box.
__device__ __forceinline__ uint32_t swz(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

// 8-bit caches: the token (0-15 within a 16-token tile) that row r of the q.K MMA holds. Rows
// 0-3, 4-7, 8-11, 12-15 hold tokens 0-3, 12-15, 4-7, 8-11: each 8-row half reads 8 distinct swizzle
// positions, and so do the halves of the p.V loads (v_tok).
__device__ __forceinline__ constexpr int tok_of_row(int r) { return r < 4 ? r : (r < 8 ? r + 8 : r - 4); }
// The token at row i of the transposed p.V byte loads: lane (g, t) then holds tokens v_tok(4t),
// v_tok(4t + 1) of the q.K row 2t (scores of rows 2t and 2t + 8) and v_tok(4t + 2), v_tok(4t + 3) of
// row 2t + 1, so the softmax weights reach the p.V operand as packed pairs.
__device__ __forceinline__ constexpr int v_tok(int i)
{
    return tok_of_row(2 * (i >> 2) + ((i >> 1) & 1) + 8 * (i & 1));
}

// Tokens of sequence s this pass streams: seq_lens[s] clamped to [0, capacity], less the
// skip_blocks[s] leading blocks of a shared-prefix suffix pass (at most the full blocks). `err`
// collects PKV_DEVERR_SEQ_LEN / PKV_DEVERR_PLAN for values that needed clamping.
__device__ __forceinline__ int stream_tokens(const DecodeParams& p, int s, int BS, int capacity, int& skip, int& err)
{
    int L = p.seq_lens[s];
    if (L < 0 || L > capacity) {
        err |= PKV_DEVERR_SEQ_LEN;
        L = L < 0 ? 0 : capacity;
    }
    skip = 0;
    if (p.skip_blocks != nullptr) {
        skip = p.skip_blocks[s];
        if (skip < 0 || skip > L / BS) {
            err |= PKV_DEVERR_PLAN;
            skip = skip < 0 ? 0 : L / BS;
        }
    }
    return L - skip * BS;
}

// prefix[s] = units (head group x UT tokens) of sequences before s, units of a sequence =
// ceil(L / UT) * groups with L the tokens the pass streams (stream_tokens, blocks of BS tokens;
// UT = BS for the warp-MMA kernel, whose unit is one block). All threads of the CTA; ends with a
// barrier. Returns the PKV_DEVERR_* bits of clamped lengths or skips. With `info`, also
// info[s] = (streamed tokens, skipped blocks) of every sequence.
__device__ __forceinline__ int build_unit_prefix(const DecodeParams& p, int* prefix, int BS, int NHG, int capacity,
                                                 int UT, int2* info = nullptr)
{
    const int tid = threadIdx.x, lane = tid & 31;
    int bad = 0;
    for (int s = tid; s < p.num_seqs; s += blockDim.x) {
        int skip;
        const int L = stream_tokens(p, s, BS, capacity, skip, bad);
        prefix[s + 1] = ((L + UT - 1) / UT) * NHG;
        if (info != nullptr)
            info[s] = make_int2(L, skip);
    }
    if (tid == 0)
        prefix[0] = 0;
    const int any_bad = __syncthreads_or(bad & PKV_DEVERR_SEQ_LEN) ? PKV_DEVERR_SEQ_LEN : 0;
    const int any_plan = __syncthreads_or(bad & PKV_DEVERR_PLAN) ? PKV_DEVERR_PLAN : 0;
    if (tid < 32) {
        int carry = 0;
        for (int base = 0; base < p.num_seqs; base += 32) {
            const int i = base + lane + 1;
            int v = (i <= p.num_seqs) ? prefix[i] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(kFullMask, v, o);
                if (lane >= o)
                    v += u;
            }
            v += carry;
            if (i <= p.num_seqs)
                prefix[i] = v;
            carry = __shfl_sync(kFullMask, v, 31);
        }
    }
    __syncthreads();
    return any_bad | any_plan;
}

// The units of a launch, in (sequence, head group, block) order, cut into chunks. Chunk c < R (R =
// the grid's CTAs) is CTA c's own: [c * P1, (c + 1) * P1), three quarters of the work shared out
// evenly. The last quarter is cut into chunks of P2 >= min_chunk units, about tail_chunks per
// CTA, which CTAs claim from a counter as they finish: SMs that stream slower take fewer of
// them, so the grid ends together. With tail_chunks = 0 (or fewer than min_units units per CTA)
// the R own chunks cover everything. Chunks are contiguous and in order: the pieces of a stream are
// chunks of(begin) .. of(end - 1), the same for every schedule.
struct Chunks {
    int R, P1, P2, C, U;
    __device__ __forceinline__ int begin(int c) const { return c < R ? c * P1 : R * P1 + (c - R) * P2; }
    __device__ __forceinline__ int end(int c) const
    {
        return min(U, c < R ? (c + 1) * P1 : R * P1 + (c - R + 1) * P2);
    }
    __device__ __forceinline__ int of(int x) const { return x < R * P1 ? x / P1 : R + (x - R * P1) / P2; }
};

__device__ __forceinline__ Chunks make_chunks(int U, int R, int tail_chunks, int min_units, int min_chunk)
{
    Chunks ch;
    ch.R = R;
    ch.U = U;
    const int per = (U + R - 1) / R;
    if (tail_chunks <= 0 || U < min_units * R) {   // static: one run per CTA
        ch.P1 = per > 0 ? per : 1;
        ch.P2 = 1;
        ch.C = R;
        return ch;
    }
    ch.P1 = (int)(3ll * U / (4ll * R));
    const int rem = U - R * ch.P1;
    const int want = (rem + R * tail_chunks - 1) / (R * tail_chunks);
    ch.P2 = want > min_chunk ? want : min_chunk;
    ch.C = R + (rem + ch.P2 - 1) / ch.P2;
    return ch;
}

// ------------------------------------------------------------------ kernel

template <class KV, class QT, int D, int BS, int G, int HG, bool PFX = false>
__global__ void __launch_bounds__(MmaCfg<KV, D, BS, G, HG, PFX>::kThreads, MmaCfg<KV, D, BS, G, HG, PFX>::kCtasPerSM)
    paged_decode_mma_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                            const DecodeParams p)
{
    using C = MmaCfg<KV, D, BS, G, HG, PFX>;
    constexpr int W = C::W;
    constexpr bool F16 = C::kF16;
    constexpr bool I8 = C::kI8;
    // lazy running max: moved only when a tile max passes it by kSlack (log2 units), so p <= 2^8
    constexpr float kSlack = kMmaRescaleSlack;
    const int S = p.stages_per_warp;   // ring depth (stages of the CTA)
    const int Hkv = p.num_kv_heads;
    const int NHG = Hkv / HG;          // head groups per sequence
    const int capacity = p.max_blocks_per_seq * BS;

    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* stages = smem;                                                    // [S][kStage], 1024-aligned
    uint64_t* full = reinterpret_cast<uint64_t*>(stages + (size_t)S * C::kStage);
    uint64_t* empty = full + S;
    int* skip = reinterpret_cast<int*>(empty + S);
    volatile int* abort_flag = skip + S;
    int* chunk_ring = const_cast<int*>(abort_flag + 1);                       // [kChunkRing] chunk ids
    int* chunk_cnt = chunk_ring + kChunkRing;                                  // [kChunkRing] warps done
    int* prefix = chunk_cnt + kChunkRing;                                      // [num_seqs + 1]

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    // the merge kernel that follows may be scheduled now; it waits for this grid before reading
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if ((smem_addr(smem) & 1023u) != 0u) {   // the 128-byte swizzle needs 1024-byte aligned stages
        if (tid == 0) {
            atomicOr(p.err, PKV_DEVERR_TIMEOUT);
            if (p.wait_prior_at_exit)
                asm volatile("griddepcontrol.wait;" ::: "memory");
        }
        return;
    }

    if (tid == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], W);
        }
        *abort_flag = 0;
        for (int i = 0; i < kChunkRing; ++i)
            chunk_cnt[i] = 0;
        fence_mbar_init();
    }
    {
        const int bad = build_unit_prefix(p, prefix, BS, NHG, capacity, BS);
        if (bad && blockIdx.x == 0 && tid == 0)
            atomicOr(p.err, bad);
    }

    const int total = prefix[p.num_seqs];
    const int nruns = gridDim.x;
    const Chunks ch = make_chunks(total, nruns, p.tail_chunks, p.tail_min_units, p.tail_min_chunk);

    // zero rows of empty sequences (one run per sequence); a prefix pass writes no rows, and a
    // suffix pass leaves the rows of sequences with shared blocks to the merge
    for (int s = blockIdx.x; !PFX && s < p.num_seqs; s += nruns) {
        if (prefix[s + 1] == prefix[s]) {
            // a new token needs a position in the sequence: seq_lens[s] >= 1 (and, in a suffix pass,
            // a block of its own)
            if (tid == 0 && p.new_k != nullptr && __ldg(p.new_slots + s) >= 0)
                atomicOr(p.err, PKV_DEVERR_SLOT);
            if (p.skip_blocks != nullptr) {
                int skipb, e = 0;
                (void)stream_tokens(p, s, BS, capacity, skipb, e);
                if (skipb > 0)
                    continue;
            }
            const int rows = p.num_heads * (p.q_len > 1 ? p.q_len : 1);
            QT* o = reinterpret_cast<QT*>(p.out) + (size_t)s * rows * D;
            for (int i = tid; i < rows * D; i += C::kThreads)
                from_float(0.f, o + i);
        }
    }

    // =========================== producer warp ===============================
    if (warp == W) {
        if (lane == 0) {
            prefetch_tensormap(&kmap);
            prefetch_tensormap(&vmap);
        }
        // chunks: this CTA's own, then tail chunks claimed one ahead (the claim's round trip
        // overlaps the current chunk's copies)
        int cur = blockIdx.x;
        int nxt = ch.C;
        if (lane == 0 && ch.C > ch.R)
            nxt = ch.R + atomicAdd(p.chunk_ctr, 1);
        bool aborted = false;
        int issued = 0;
        int k = 0;                 // stages issued so far (ring position)
        int published = 0;         // chunks announced to the consumers
        while (cur < ch.C && !aborted) {
            const int cb = ch.begin(cur);
            const int nunits = ch.end(cur) - cb;
            if (nunits > 0) {
                if (lane == 0)
                    chunk_ring[published % kChunkRing] = cur;   // read after this chunk's first stage fills
                ++published;
            }
            // lane l resolves unit (batch + l): pool row of its head group, or -1 for a bad block
            // id; `app` is the stream (sequence * NHG + head group) whose new token lands in this
            // unit (its last block) when the launch also appends, else -1
            auto locate = [&](int kk, int& app) -> int {
                app = -1;
                if (kk >= nunits)
                    return -1;
                const int x = cb + kk;
                const int s = find_seq(prefix, p.num_seqs, x);
                const int nb = (prefix[s + 1] - prefix[s]) / NHG;
                const int r = x - prefix[s];
                const int hg = r / nb, j = r - hg * nb;
                if (p.new_k != nullptr && j == nb - 1)
                    app = s * NHG + hg;
                int skipb = 0;
                if (p.skip_blocks != nullptr) {   // a suffix pass starts past the shared blocks
                    int e = 0;
                    (void)stream_tokens(p, s, BS, capacity, skipb, e);
                }
                const int phys = __ldg(p.block_tables + (long long)s * p.max_blocks_per_seq + skipb + j);
                if (phys < 0 || phys >= p.num_blocks) {
                    atomicOr(p.err, PKV_DEVERR_BLOCK_ID);
                    return -1;
                }
                return (phys * Hkv + hg * HG) * BS;
            };
            int cur_app, ahead_app;
            int cur_row = locate(lane, cur_app), ahead = locate(32 + lane, ahead_app);
            for (int k0 = 0; k0 < nunits && !aborted; k0 += 32) {
                if (k0 > 0) {
                    cur_row = ahead;
                    cur_app = ahead_app;
                    ahead = locate(k0 + 32 + lane, ahead_app);
                }
                const int cnt = min(32, nunits - k0);
                for (int i = 0; i < cnt; ++i) {
                    const int row = __shfl_sync(kFullMask, cur_row, i);
                    const int app = __shfl_sync(kFullMask, cur_app, i);
                    if (app >= 0)   // the decode-step append of this stream, before its last block is read
                        append_new_token_impl<KV>(p, app / NHG, (app % NHG) * HG, HG, D, BS, lane,
                                                  row < 0 ? -1 : row / (Hkv * BS));
                    if (lane == 0 && !aborted) {
                        const int st = k % S;
                        if (*abort_flag) {
                            aborted = true;
                        } else if (k >= S && !mbar_wait_bounded(&empty[st], ((k / S) - 1) & 1)) {
                            aborted = true;
                            *abort_flag = 1;
                            atomicOr(p.err, PKV_DEVERR_TIMEOUT);
                        } else if (p.withheld_unit != 0 && cb + k0 + i == p.withheld_unit - 1) {
                            aborted = true;   // test hook: this stage never fills; issue nothing more
                        } else if (row < 0) {
                            skip[st] = 1;
                            mbar_arrive(&full[st]);
                            issued = k + 1;
                        } else {
                            skip[st] = 0;
                            uint8_t* dst = stages + (size_t)st * C::kStage;
                            mbar_arrive_expect_tx(&full[st], C::kStage);
#pragma unroll
                            for (int bx = 0; bx < C::kBoxes; ++bx) {
                                tma_load_2d(dst + bx * C::kBoxBytes, &kmap, bx * C::kBoxCols, row, &full[st]);
                                tma_load_2d(dst + C::kHalf + bx * C::kBoxBytes, &vmap, bx * C::kBoxCols, row,
                                            &full[st]);
                            }
                            issued = k + 1;
                        }
                    }
                    ++k;
                }
                aborted = __shfl_sync(kFullMask, aborted ? 1 : 0, 0) != 0;
            }
            cur = __shfl_sync(kFullMask, nxt, 0);
            if (lane == 0 && cur < ch.C)
                nxt = ch.R + atomicAdd(p.chunk_ctr, 1);
        }
        // end of the work: a stage without bytes whose chunk id is -1 tells the consumers
        if (lane == 0 && !aborted) {
            const int st = k % S;
            if (k >= S && !mbar_wait_bounded(&empty[st], ((k / S) - 1) & 1)) {
                aborted = true;
                *abort_flag = 1;
                atomicOr(p.err, PKV_DEVERR_TIMEOUT);
            } else {
                chunk_ring[published % kChunkRing] = -1;
                skip[st] = 1;
                mbar_arrive(&full[st]);
            }
        }
        if (lane == 0 && aborted) {
            for (int kk = max(0, issued - S); kk < issued; ++kk)
                (void)mbar_wait_bounded(&full[kk % S], (kk / S) & 1);
        }
        return;
    }

    // =========================== consumer warps ==============================
    const int g = lane >> 2;   // MMA row group
    const int t = lane & 3;    // MMA column pair


    int k = 0;                 // stages consumed so far (ring position)
    for (int ordinal = 0;; ++ordinal) {
        // the first stage of the CTA's next chunk carries the chunk's id (-1: no more work)
        {
            const int st = k % S;
            const bool ok = !*abort_flag && mbar_wait_bounded(&full[st], (k / S) & 1);
            if (!__all_sync(kFullMask, ok)) {
                if (lane == 0 && !*abort_flag) {
                    *abort_flag = 1;
                    atomicOr(p.err, PKV_DEVERR_TIMEOUT);
                }
                break;
            }
        }
        const int cur = chunk_ring[ordinal % kChunkRing];
        if (cur < 0 || cur >= ch.C)
            break;
        const int run_end = ch.end(cur);
        int x = ch.begin(cur);
        while (x < run_end) {
            const int s = find_seq(prefix, p.num_seqs, x);
            const int nb = (prefix[s + 1] - prefix[s]) / NHG;
            const int hg = (x - prefix[s]) / nb;
            const int stream_begin = prefix[s] + hg * nb;
            const int stream_end = stream_begin + nb;
            const int seg_end = min(run_end, stream_end);
            const int head = hg * HG + warp / C::kNT;   // this warp's KV head
            const int tile = warp % C::kNT;             // prefix pass: this warp's 8 of the 32 columns
            int skipb = 0, lerr = 0;
            const int L = stream_tokens(p, s, BS, capacity, skipb, lerr);
            const int QL = p.q_len > 1 ? p.q_len : 1;
            const int Gq = p.num_heads / p.num_kv_heads;
            // FP8 per-head scales (when given): this head's into the score and output factors
            const float qk_scale = p.k_head_scales ? p.q_scale * __ldg(p.k_head_scales + head) : p.q_scale;
            const float out_scale = p.v_head_scales ? p.v_scale * __ldg(p.v_head_scales + head) : p.v_scale;
            // Query column c (0..7) of this warp: its row of q / out, and how many of the stream's
            // tokens it sees. Decode: column c is new token c / Gq of q_len and sees the tokens before
            // position L - q_len + 1 + c / Gq (all L when q_len = 1); columns >= G are padding.
            // Prefix pass: column tile * 8 + c is query head (.. % Gq) of member (.. / Gq) of group s,
            // which sees its own shared blocks of the group's row; columns past the members: padding.
            auto column = [&](int c, size_t& row) -> int {
                row = 0;
                if constexpr (PFX) {
                    const int cg = tile * 8 + c, mem = cg / Gq;
                    const int off = p.pfx_offsets[s], cnt = p.pfx_offsets[s + 1] - off;
                    if (mem >= cnt || mem >= p.pfx_max_group)
                        return 0;
                    const int seq = p.pfx_members[off + mem];
                    if (seq < 0 || seq >= p.pfx_num_seqs)
                        return 0;
                    row = (size_t)seq * p.num_heads + (size_t)head * Gq + (cg - mem * Gq);
                    const int lim = p.pfx_shared[seq] * BS;
                    return lim < 0 ? 0 : (lim < L ? lim : L);
                } else {
                    if (c >= G)
                        return 0;
                    row = query_row(p, s, head, c);
                    return L - QL + 1 + c / Gq;
                }
            };
            size_t row_g, row0, row1;
            const int lim_g = column(g, row_g);
            const int lim0 = column(2 * t, row0);
            const int lim1 = column(2 * t + 1, row1);
            const bool qcol = PFX ? lim_g > 0 : g < G;   // this lane holds a real column g of Q^T
            if constexpr (PFX) {
                if (tile == 0 && lane == 0) {
                    const int off = p.pfx_offsets[s], cnt = p.pfx_offsets[s + 1] - off;
                    bool bad = cnt > p.pfx_max_group;
                    for (int i = 0; i < cnt && i < p.pfx_max_group; ++i) {
                        const int seq = p.pfx_members[off + i];
                        bad |= seq < 0 || seq >= p.pfx_num_seqs || p.pfx_shared[seq] * BS > L;
                    }
                    if (bad)
                        atomicOr(p.err, PKV_DEVERR_PLAN);
                }
            }

            // Q^T as the B operand: b0 = (k: d pair, n: query column g); columns g >= G are zero.
            uint32_t qb[C::kKS][2];
            float qk0 = qk_scale, qk1 = qk_scale;   // score factors of this lane's columns 2t, 2t+1
            if constexpr (F16) {
                // 8-bit caches: column g of Q^T times a power of two sigma_g, 1 / sigma_g going into
                // the column's score factor. f16 MMA: max |q| * sigma_g < 2^14 (exact for a bf16 q at
                // any magnitude), k order permuted to match the widened A fragments:
                // qb[ks] = (d 16ks + 4t, +1 | +2, +3). Integer MMA (INT8): max |q| * sigma_g < 2^13,
                // rounded to x = 128 hi + lo, qb[kk] hi and qb[D/32 + kk] lo as s8, b0 = d 32kk + 4t
                // .. +3, b1 = d 32kk + 16 + 4t .. +3.
                constexpr int K8 = D / 32;
                const QT* qp = reinterpret_cast<const QT*>(p.q) + row_g * D;
                float f[K8][2][4];
                float mx = 0.f;
#pragma unroll
                for (int kk = 0; kk < K8; ++kk)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        if (qcol)
                            load_q<4>(qp + kk * 32 + hh * 16 + 4 * t, f[kk][hh]);
                        else
                            f[kk][hh][0] = f[kk][hh][1] = f[kk][hh][2] = f[kk][hh][3] = 0.f;
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            mx = fmaxf(mx, fabsf(f[kk][hh][i]));
                    }
                mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, 2));
                // mx < 2^(E - 126) with E its biased exponent; sigma = 2^(140 - E) (f16) or
                // 2^(139 - E) (s8), kept normal both ways
                int se = 127;
                if (mx > 0.f) {
                    se = 127 + (I8 ? 139 : 140) - (int)((__float_as_uint(mx) >> 23) & 0xffu);
                    se = se < 2 ? 2 : (se > 252 ? 252 : se);
                }
                const float sig = __uint_as_float((uint32_t)se << 23);
                const float inv_sig = __uint_as_float((uint32_t)(254 - se) << 23);
#pragma unroll
                for (int kk = 0; kk < K8; ++kk)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        if constexpr (I8) {
                            const float v[4] = {f[kk][hh][0] * sig, f[kk][hh][1] * sig, f[kk][hh][2] * sig,
                                                f[kk][hh][3] * sig};
                            split_s8x4(v, qb[kk][hh], qb[K8 + kk][hh]);
                        } else {
                            qb[2 * kk + hh][0] = pack2<true>(f[kk][hh][0] * sig, f[kk][hh][1] * sig);
                            qb[2 * kk + hh][1] = pack2<true>(f[kk][hh][2] * sig, f[kk][hh][3] * sig);
                        }
                    }
                qk0 = qk_scale * __shfl_sync(kFullMask, inv_sig, (2 * t) * 4);
                qk1 = qk_scale * __shfl_sync(kFullMask, inv_sig, (2 * t + 1) * 4);
            } else {
                const QT* qp = reinterpret_cast<const QT*>(p.q) + row_g * D;
#pragma unroll
                for (int ks = 0; ks < C::kKS; ++ks) {
                    if (qcol) {
                        qb[ks][0] = __ldg(reinterpret_cast<const uint32_t*>(qp + ks * 16 + 2 * t));
                        qb[ks][1] = __ldg(reinterpret_cast<const uint32_t*>(qp + ks * 16 + 2 * t + 8));
                    } else {
                        qb[ks][0] = qb[ks][1] = 0u;
                    }
                }
            }
            float o[C::kDT][4];
#pragma unroll
            for (int dt = 0; dt < C::kDT; ++dt)
                o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
            float m[2] = {-INFINITY, -INFINITY};   // running reference for heads 2t, 2t+1
            float l[2] = {0.f, 0.f};

            for (; x < seg_end; ++x, ++k) {
                const int st = k % S;
                bool ok = !*abort_flag && mbar_wait_bounded(&full[st], (k / S) & 1);
                if (__any_sync(kFullMask, !ok)) {
                    if (lane == 0 && !*abort_flag) {
                        *abort_flag = 1;
                        atomicOr(p.err, PKV_DEVERR_TIMEOUT);
                    }
                    ok = false;
                }
                const int jb = x - stream_begin;         // logical block
                const int valid = min(BS, L - jb * BS);
                bool released = false;
                if (ok && skip[st] == 0 && valid > 0) {
                    const uint32_t kbase = smem_addr(stages + (size_t)st * C::kStage);
                    const uint32_t vbase = kbase + C::kHalf;
                    const int r0 = (warp / C::kNT) * BS;   // this warp's KV head's first box row
#pragma unroll
                    for (int tt = 0; tt < C::kTT; ++tt) {
                        // ---- S^T = K Q^T : 16 tokens x 8 heads
                        float sc[4] = {0.f, 0.f, 0.f, 0.f};
                        float sd[4] = {0.f, 0.f, 0.f, 0.f};   // second accumulator: halves the MMA dependency chain
                        const int mi = lane >> 3, rr = lane & 7;
                        // 8-bit caches: MMA row r of the tile holds token tok_of_row(r), so that this
                        // lane's scores (rows g, g + 8) are the token pair its P^T value carries
                        const int krow = r0 + tt * 16 + (F16 ? tok_of_row((mi & 1) * 8 + rr) : (mi & 1) * 8 + rr);
                        if constexpr (I8) {
                            // matrices (MMA rows 0-7 | 8-15) x (chunk 2kk | 2kk+1): the m16n8k32 A fragment
                            // of 16 tokens x d 32kk .. 32kk+31 of INT8 codes as it lies in the stage, against
                            // q's s8 hi and lo: exact int32 sums, combined as 128 hi + lo
                            int ih[4] = {0, 0, 0, 0}, il[4] = {0, 0, 0, 0};
#pragma unroll
                            for (int kk = 0; kk < D / 32; ++kk) {
                                uint32_t a[4];
                                ldsm_x4(kbase + swz(krow, 2 * kk + (mi >> 1)), a);
                                mma_16832_s8(ih, a, qb[kk][0], qb[kk][1]);
                                mma_16832_s8(il, a, qb[D / 32 + kk][0], qb[D / 32 + kk][1]);
                            }
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                sc[i] = (float)(ih[i] * 128 + il[i]);
                        } else if constexpr (F16) {
#pragma unroll
                            for (int ks = 0; ks < C::kKS; ks += 2) {
                                // matrices: (MMA rows 0-7 | 8-15) x (chunk ks | ks+1), 8 tokens x 16 codes each;
                                // each lane's 4 codes of a row widen to the A pairs (d 4t, 4t+1 | 4t+2, 4t+3)
                                uint32_t r[4];
                                ldsm_x4(kbase + swz(krow, ks + (mi >> 1)), r);
#pragma unroll
                                for (int h2 = 0; h2 < 2; ++h2) {
                                    uint32_t a[4];
                                    widen_halves<KV>(r[2 * h2], a[0], a[2]);
                                    widen_halves<KV>(r[2 * h2 + 1], a[1], a[3]);
                                    mma_16816<true>(h2 ? sd : sc, a, qb[ks + h2][0], qb[ks + h2][1]);
                                }
                            }
                        } else {
#pragma unroll
                            for (int ks = 0; ks < C::kKS; ++ks) {
                                // matrices: (tok 0-7, d 0-7), (tok 8-15, d 0-7), (tok 0-7, d 8-15), (tok 8-15, d 8-15)
                                const int box = ks / 4, chunk = (ks % 4) * 2 + (mi >> 1);
                                uint32_t a[4];
                                ldsm_x4(kbase + box * C::kBoxBytes + swz(krow, chunk), a);
                                mma_16816<false>((ks & 1) ? sd : sc, a, qb[ks][0], qb[ks][1]);
                            }
                        }
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            sc[i] += sd[i];
                        // V fragments of this tile into registers; after the block's last tile the
                        // stage goes back to the producer before the softmax and p.V arithmetic
                        uint32_t vf[C::kDT * 4 / (F16 ? 2 : 1)];
                        if constexpr (F16) {
#pragma unroll
                            for (int dt = 0; dt < C::kDT; dt += 2) {
                                // matrices: the tile's 16 tokens x chunk dt | dt + 1 (d 16dt .. 16dt + 31),
                                // transposed: r[0] = d 16dt + g of tokens v_tok(4t .. 4t + 3), r[1] = d +8,
                                // r[2], r[3] the same for chunk dt + 1
                                const int row = r0 + tt * 16 + v_tok(lane & 15);
                                uint32_t r[4];
                                ldsm_b8_x2_t(vbase + swz(row, dt + (lane >> 4)), r);
#pragma unroll
                                for (int i = 0; i < 4; ++i)
                                    vf[2 * dt + i] = r[i];
                            }
                        } else {
#pragma unroll
                            for (int dt = 0; dt < C::kDT; ++dt) {
                                // matrices: (d 0-7, tok 0-7), (d 8-15, tok 0-7), (d 0-7, tok 8-15), (d 8-15, tok 8-15)
                                const int row = r0 + tt * 16 + (mi >> 1) * 8 + rr;
                                const int box = dt / 4, chunk = (dt % 4) * 2 + (mi & 1);
                                uint32_t r[4];
                                ldsm_x4_t(vbase + box * C::kBoxBytes + swz(row, chunk), r);
#pragma unroll
                                for (int i = 0; i < 4; ++i)
                                    vf[4 * dt + i] = r[i];
                            }
                        }
                        if (tt == C::kTT - 1) {
                            __syncwarp();
                            if (lane == 0)
                                mbar_arrive(&empty[st]);
                            released = true;
                        }
                        // sc: (token g | g+8) x (heads 2t, 2t+1), in log2 units after the scale
                        // positions in the sequence of rows g and g + 8
                        const int tok0 = jb * BS + tt * 16 + (F16 ? tok_of_row(g) : g);
                        const int tok8 = jb * BS + tt * 16 + (F16 ? tok_of_row(g + 8) : g + 8);
                        sc[0] = (tok0 < lim0) ? sc[0] * qk0 : -INFINITY;
                        sc[1] = (tok0 < lim1) ? sc[1] * qk1 : -INFINITY;
                        sc[2] = (tok8 < lim0) ? sc[2] * qk0 : -INFINITY;
                        sc[3] = (tok8 < lim1) ? sc[3] * qk1 : -INFINITY;
                        // The reference moves only when some score passes it by the slack; each lane
                        // tests its own scores first, so the butterfly max runs only when one does
                        // (same result as reducing first: the tile max passes iff some lane's does).
                        float bm0 = fmaxf(sc[0], sc[2]), bm1 = fmaxf(sc[1], sc[3]);
                        if (__any_sync(kFullMask, bm0 > m[0] + kSlack || bm1 > m[1] + kSlack)) {
#pragma unroll
                            for (int off = 4; off < 32; off <<= 1) {
                                bm0 = fmaxf(bm0, __shfl_xor_sync(kFullMask, bm0, off));
                                bm1 = fmaxf(bm1, __shfl_xor_sync(kFullMask, bm1, off));
                            }
                            const bool up0 = bm0 > m[0] + kSlack, up1 = bm1 > m[1] + kSlack;
                            const float n0 = up0 ? bm0 : m[0], n1 = up1 ? bm1 : m[1];
                            const float a0 = up0 ? fast_exp2(m[0] - n0) : 1.f, a1 = up1 ? fast_exp2(m[1] - n1) : 1.f;
                            m[0] = n0;
                            m[1] = n1;
                            l[0] *= a0;
                            l[1] *= a1;
#pragma unroll
                            for (int dt = 0; dt < C::kDT; ++dt) {
                                o[dt][0] *= a0;
                                o[dt][1] *= a1;
                                o[dt][2] *= a0;
                                o[dt][3] *= a1;
                            }
                        }
                        float pr[4];
                        pr[0] = (sc[0] == -INFINITY) ? 0.f : fast_exp2(sc[0] - m[0]);
                        pr[1] = (sc[1] == -INFINITY) ? 0.f : fast_exp2(sc[1] - m[1]);
                        pr[2] = (sc[2] == -INFINITY) ? 0.f : fast_exp2(sc[2] - m[0]);
                        pr[3] = (sc[3] == -INFINITY) ? 0.f : fast_exp2(sc[3] - m[1]);
                        l[0] += pr[0] + pr[2];
                        l[1] += pr[1] + pr[3];
                        const int srcA = (2 * t) * 4 + (g >> 1), srcB = (2 * t + 1) * 4 + (g >> 1);
                        uint32_t pb0, pb1;
                        {
                            // ---- P^T as the B operand: b0 = (tokens 2t, 2t+1; head g), b1 = (tokens 2t+8, 2t+9; head g)
                            const uint32_t X = pack2<F16>(pr[0], pr[2]);   // head 2t:   tokens g, g+8
                            const uint32_t Y = pack2<F16>(pr[1], pr[3]);   // head 2t+1: tokens g, g+8
                            const uint32_t xa = __shfl_sync(kFullMask, X, srcA), ya = __shfl_sync(kFullMask, Y, srcA);
                            const uint32_t xb = __shfl_sync(kFullMask, X, srcB), yb = __shfl_sync(kFullMask, Y, srcB);
                            const uint32_t va = (g & 1) ? ya : xa, vb = (g & 1) ? yb : xb;
                            if constexpr (F16) {
                                // 8-bit caches: lane 4(2t) + g/2 holds tokens v_tok(4t), v_tok(4t + 1) of
                                // head g, lane 4(2t + 1) + g/2 tokens v_tok(4t + 2), v_tok(4t + 3)
                                pb0 = qcol ? va : 0u;
                                pb1 = qcol ? vb : 0u;
                            } else {
                                pb0 = qcol ? __byte_perm(va, vb, 0x5410) : 0u;
                                pb1 = qcol ? __byte_perm(va, vb, 0x7632) : 0u;
                            }
                        }
                        // ---- O^T += V^T P^T : head_dim x 8 heads, k = the tile's 16 tokens
                        const bool partial = valid < tt * 16 + 16;
                        if constexpr (F16) {
                            // byte e of a V register is token v_tok(4t + e): in a partial tile the codes
                            // past the sequence's end are cleared (stale codes may be NaN); full tiles
                            // run a copy of the loop without the masks
                            auto pv = [&](auto masked, uint32_t keep) {
#pragma unroll
                                for (int dt = 0; dt < C::kDT; dt += 2) {
#pragma unroll
                                    for (int h2 = 0; h2 < 2; ++h2) {
                                        // d 16(dt + h2) + g (row g) and + 8 (row g + 8); k 2t, 2t+1 are tokens
                                        // v_tok(4t), v_tok(4t + 1) (bytes 0, 1), k 2t+8, 2t+9 bytes 2, 3
                                        uint32_t rg = vf[2 * dt + 2 * h2], rg8 = vf[2 * dt + 2 * h2 + 1];
                                        if constexpr (decltype(masked)::value) {
                                            rg &= keep;
                                            rg8 &= keep;
                                        }
                                        uint32_t a[4];
                                        widen_halves<KV>(rg, a[0], a[2]);
                                        widen_halves<KV>(rg8, a[1], a[3]);
                                        mma_16816<true>(o[dt + h2], a, pb0, pb1);
                                    }
                                }
                            };
                            if (partial) {
                                uint32_t keep = 0u;
#pragma unroll
                                for (int e = 0; e < 4; ++e)
                                    keep |= (tt * 16 + v_tok(4 * t + e) < valid) ? 0xffu << (8 * e) : 0u;
                                pv(std::true_type{}, keep);
                            } else {
                                pv(std::false_type{}, 0u);
                            }
                        } else {
#pragma unroll
                            for (int dt = 0; dt < C::kDT; ++dt) {
                                uint32_t a[4] = {vf[4 * dt], vf[4 * dt + 1], vf[4 * dt + 2], vf[4 * dt + 3]};
                                if (partial) {
                                    const int tk = tt * 16 + 2 * t;
                                    const uint32_t m01 = (tk < valid ? 0x0000ffffu : 0u) | (tk + 1 < valid ? 0xffff0000u : 0u);
                                    const uint32_t m89 = (tk + 8 < valid ? 0x0000ffffu : 0u) | (tk + 9 < valid ? 0xffff0000u : 0u);
                                    a[0] &= m01;
                                    a[1] &= m01;
                                    a[2] &= m89;
                                    a[3] &= m89;
                                }
                                mma_16816<false>(o[dt], a, pb0, pb1);
                            }
                        }
                    }
                }
                if (!released) {
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&empty[st]);
                }
            }

            // ---- end of this warp's segment: l over the 8 row groups, then write or merge
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                l[0] += __shfl_xor_sync(kFullMask, l[0], off);
                l[1] += __shfl_xor_sync(kFullMask, l[1], off);
            }
            const int first_run = ch.of(stream_begin);   // chunks holding pieces of this stream
            const int last_run = ch.of(stream_end - 1);
            const int stream = s * NHG + hg;
            // element (head column c, row d) of this lane's accumulators
            auto d_of = [&](int dt, int half) -> int {
                return dt * 16 + g + 8 * half;
            };
            // a whole stream writes `out`; pieces of split streams, every stream of a prefix pass and
            // the suffix of a sequence with shared blocks leave (o, m, l) for the merge
            if (first_run == last_run && !PFX && skipb == 0) {
                QT* out0 = reinterpret_cast<QT*>(p.out) + row0 * D;
                QT* out1 = reinterpret_cast<QT*>(p.out) + row1 * D;
                const float inv0 = l[0] > 0.f ? out_scale / l[0] : 0.f;
                const float inv1 = l[1] > 0.f ? out_scale / l[1] : 0.f;
#pragma unroll
                for (int dt = 0; dt < C::kDT; ++dt)
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const int d = d_of(dt, half);
                        if (2 * t < G)
                            from_float(o[dt][2 * half] * inv0, out0 + d);
                        if (2 * t + 1 < G)
                            from_float(o[dt][2 * half + 1] * inv1, out1 + d);
                    }
            } else {
                float* part = p.partials + ((size_t)(cur + stream) * W + warp) * p.slot_floats;
#pragma unroll
                for (int dt = 0; dt < C::kDT; ++dt)
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const int d = d_of(dt, half);
                        if (2 * t < G)
                            part[(2 * t) * D + d] = o[dt][2 * half];
                        if (2 * t + 1 < G)
                            part[(2 * t + 1) * D + d] = o[dt][2 * half + 1];
                    }
                if (g == 0) {
                    if (2 * t < G) {
                        part[G * D + 2 * t] = m[0];
                        part[G * D + G + 2 * t] = l[0];
                    }
                    if (2 * t + 1 < G) {
                        part[G * D + 2 * t + 1] = m[1];
                        part[G * D + G + 2 * t + 1] = l[1];
                    }
                }
            }
        }
        // The chunk is done for this warp. The last of the W consumer warps to get here stamps it:
        // every lane's writes are made visible device-wide first, so a merge that sees the stamp
        // sees the pieces.
        if (p.chunk_done != nullptr) {
            __threadfence();
            __syncwarp();
            if (lane == 0) {
                int* cnt = &chunk_cnt[ordinal % kChunkRing];
                if (atomicAdd(cnt, 1) == W - 1) {
                    *cnt = 0;
                    __threadfence();
                    const unsigned long long v = chunk_stamp(p.epoch);
                    asm volatile("st.release.gpu.global.b64 [%0], %1;" ::"l"(p.chunk_done + cur), "l"(v) : "memory");
                }
            }
            __syncwarp();
        }
    }
    // a suffix pass launched behind a prefix pass completes only after it (see the launcher)
    if (p.wait_prior_at_exit && tid == 0)
        asm volatile("griddepcontrol.wait;" ::: "memory");
}

// One piece of a query column: its o (D floats), m and l.
struct PieceRef {
    const float* o;
    const float* m;
    const float* l;
};

// Log-sum-exp combination of the n pieces of one query column into dst (one warp; lane i owns
// floats 4i .. 4i + 3 of the D): out = sum_i e^{m_i - M} o_i / sum_i e^{m_i - M} l_i, times
// out_scale. Every lane loads one piece's (m, l), then the o slices stream in eight pieces at a
// time, so a column split into many pieces costs a few round trips, not one per piece.
template <class QT, int D, class Piece>
__device__ __forceinline__ void merge_column(int n, Piece piece, float out_scale, QT* dst, int lane)
{
    const bool mine = 4 * lane < D;
    float M = -INFINITY, Lsum = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c0 = 0; c0 < n; c0 += 32) {
        const int cnt = min(32, n - c0);
        float mi = -INFINITY, li = 0.f;
        if (lane < cnt) {
            const PieceRef r = piece(c0 + lane);
            mi = __ldcg(r.m);
            li = __ldcg(r.l);
        }
        float mx = mi;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1)
            mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, off));
        const float Mn = fmaxf(M, mx);
        if (Mn == -INFINITY)
            continue;                                   // no token in any of these pieces (warp-uniform)
        const float rescale = M == -INFINITY ? 0.f : fast_exp2(M - Mn);
        Lsum *= rescale;
        acc.x *= rescale;
        acc.y *= rescale;
        acc.z *= rescale;
        acc.w *= rescale;
        M = Mn;
        const float w = mi == -INFINITY ? 0.f : fast_exp2(mi - M);
        float lw = w * li;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1)
            lw += __shfl_xor_sync(kFullMask, lw, off);
        Lsum += lw;
        for (int j = 0; j < cnt; j += 8) {
            float4 v[8];
            float wu[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                wu[u] = __shfl_sync(kFullMask, w, (j + u) & 31);
                v[u] = (j + u < cnt && mine) ? __ldcg(reinterpret_cast<const float4*>(piece(c0 + j + u).o) + lane)
                                             : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                acc.x = fmaf(wu[u], v[u].x, acc.x);
                acc.y = fmaf(wu[u], v[u].y, acc.y);
                acc.z = fmaf(wu[u], v[u].z, acc.z);
                acc.w = fmaf(wu[u], v[u].w, acc.w);
            }
        }
    }
    if (mine) {
        const float inv = Lsum > 0.f ? out_scale / Lsum : 0.f;
        QT* o = dst + 4 * lane;
        from_float(acc.x * inv, o);
        from_float(acc.y * inv, o + 1);
        from_float(acc.z * inv, o + 2);
        from_float(acc.w * inv, o + 3);
    }
}

// Merge of query column gq of KV head (stream's head group) * HG + w of sequence s, whose stream
// left pieces in chunks first_chunk .. first_chunk + n - 1 (slot (chunk + stream) * HG + w).
template <class QT, int D, int G, int HG>
__device__ __forceinline__ void merge_split(const DecodeParams& p, int s, int stream, int first_chunk, int n, int NHG,
                                           int w, int gq, int lane)
{
    const int head = (stream - s * NHG) * HG + w;
    const float out_scale = p.v_head_scales ? p.v_scale * __ldg(p.v_head_scales + head) : p.v_scale;
    auto piece = [&](int i) -> PieceRef {
        const float* b = p.partials + ((size_t)(first_chunk + i + stream) * HG + w) * p.slot_floats;
        return PieceRef{b + gq * D, b + G * D + gq, b + G * D + G + gq};
    };
    merge_column<QT, D>(n, piece, out_scale, reinterpret_cast<QT*>(p.out) + query_row(p, s, head, gq) * D, lane);
}


// Merge of the streams the decode kernel split across chunks: one warp per (stream, KV head of
// its group, query column), launched behind the decode kernel as a programmatic dependent launch.
// The prefix is built while the decode kernel still runs (it reads only seq_lens). With chunk
// completion stamps (DecodeParams::chunk_done) each split stream is merged once its chunks are
// stamped, overlapping the decode grid's tail; otherwise griddepcontrol.wait holds until the
// decode grid has finished and its partials are visible.
constexpr int kMergeThreads = 128;

// UT: tokens per unit of the decode kernel (the block size for the warp-MMA kernel, 128 for the
// tcgen05 kernel).
template <class QT, int D, int BS, int G, int HG, int UT = BS>
__global__ void __launch_bounds__(kMergeThreads) paged_decode_merge_kernel(const DecodeParams p, int decode_runs)
{
    extern __shared__ int prefix[];   // [num_seqs + 1]
    const int NHG = p.num_kv_heads / HG;
    (void)build_unit_prefix(p, prefix, BS, NHG, p.max_blocks_per_seq * BS, UT);
    // With completion stamps, a split stream is merged as soon as the chunks holding its pieces
    // carry this call's stamp, while the decode grid still runs; without, after the whole grid.
    const bool stamped = p.chunk_done != nullptr;
    if (!stamped)
        asm volatile("griddepcontrol.wait;" ::: "memory");
    const int total = prefix[p.num_seqs];
    const int lane = threadIdx.x & 31;
    if (total > 0) {
        const Chunks ch = make_chunks(total, decode_runs, p.tail_chunks, p.tail_min_units, p.tail_min_chunk);
        const unsigned long long want = chunk_stamp(p.epoch);
        const int warps = gridDim.x * (kMergeThreads / 32);
        const int items = p.num_seqs * NHG * HG * G;
        for (int it = blockIdx.x * (kMergeThreads / 32) + (threadIdx.x >> 5); it < items; it += warps) {
            const int gq = it % G, sw = it / G;
            const int stream = sw / HG, w = sw - stream * HG;
            const int s = stream / NHG, hg = stream - s * NHG;
            const int nb = (prefix[s + 1] - prefix[s]) / NHG;
            if (nb == 0)
                continue;
            const int sb = prefix[s] + hg * nb;
            const int first_run = ch.of(sb), last_run = ch.of(sb + nb - 1);
            if (first_run == last_run)
                continue;
            if (stamped) {
                // every chunk of the stream stamped (a bounded wait; a chunk whose CTA gave up is
                // never stamped, and the call has flagged that already)
                bool ok = true;
                for (int c = first_run + lane; c <= last_run; c += 32) {
                    const uint64_t t0 = global_ns();
                    for (uint32_t polls = 0;; ++polls) {
                        unsigned long long v;
                        asm volatile("ld.acquire.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p.chunk_done + c) : "memory");
                        if (v == want)
                            break;
                        if (polls >= kWaitLimitPolls || ((polls & 15u) == 15u && global_ns() - t0 > kWaitLimitNs)) {
                            ok = false;
                            break;
                        }
                        __nanosleep(200);
                    }
                    if (!ok)
                        break;
                }
                __threadfence();
                if (!__all_sync(kFullMask, ok)) {
                    if (lane == 0)
                        atomicOr(p.err, PKV_DEVERR_TIMEOUT);
                    continue;
                }
            }
            merge_split<QT, D, G, HG>(p, s, stream, first_run, last_run - first_run + 1, NHG, w, gq, lane);
        }
    }
    // the decode grid is done claiming: the counter is ready for the next call
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        if (stamped)
            asm volatile("griddepcontrol.wait;" ::: "memory");
        *p.chunk_ctr = 0;
    }
}

// Merge of a shared-prefix decode, launched behind the suffix pass as a programmatic dependent
// launch (the suffix pass completes only after the prefix pass, so the wait covers both).
// (a) Every (member of a group with shared blocks, KV head h, query head gq), one warp each: the
//     prefix pass's pieces of column member * Gq + gq of stream (group, h) and the suffix pass's
//     pieces of the member's stream, log-sum-exp combined into out.
// (b) Sequences without shared blocks whose stream the suffix pass split: merge_split, as after a
//     plain decode.
// ps: the suffix pass's parameters (skip_blocks = the plan's shared blocks); pp: the prefix
// pass's (its "sequences" are the groups). Shared memory: both unit prefixes.
template <class QT, int D, int BS, int G, int HG>
__global__ void __launch_bounds__(kMergeThreads)
    paged_decode_prefix_merge_kernel(const DecodeParams ps, const DecodeParams pp, int runs_s, int runs_p)
{
    extern __shared__ int smem_prefix[];
    int* prefix_s = smem_prefix;                     // [num_seqs + 1]
    int* prefix_p = smem_prefix + ps.num_seqs + 1;   // [num_groups + 1]
    const int Hkv = ps.num_kv_heads, NHG = Hkv / HG, Gq = ps.num_heads / Hkv;
    const int capacity = ps.max_blocks_per_seq * BS;
    (void)build_unit_prefix(ps, prefix_s, BS, NHG, capacity, BS);
    (void)build_unit_prefix(pp, prefix_p, BS, Hkv, capacity, BS);
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (blockIdx.x == 0 && threadIdx.x == 0) {   // both passes are done claiming
        *ps.chunk_ctr = 0;
        *pp.chunk_ctr = 0;
    }
    const int total_s = prefix_s[ps.num_seqs], total_p = prefix_p[pp.num_seqs];
    const Chunks ch_s = make_chunks(total_s, runs_s, ps.tail_chunks, ps.tail_min_units, ps.tail_min_chunk);
    const Chunks ch_p = make_chunks(total_p, runs_p, pp.tail_chunks, pp.tail_min_units, pp.tail_min_chunk);
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (kMergeThreads / 32);
    const int wid = blockIdx.x * (kMergeThreads / 32) + (threadIdx.x >> 5);

    // (a) members of groups
    const int members = pp.num_seqs > 0 ? pp.pfx_offsets[pp.num_seqs] : 0;   // no groups: no plan arrays
    const int items_a = members * Hkv * Gq;
    for (int it = wid; it < items_a; it += warps) {
        const int mm = it / (Hkv * Gq), rem = it - mm * (Hkv * Gq);
        const int h = rem / Gq, gq = rem - h * Gq;
        int lo = 0, hi = pp.num_seqs;                 // group of member mm: offsets[gi] <= mm < offsets[gi + 1]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (pp.pfx_offsets[mid] <= mm)
                lo = mid;
            else
                hi = mid;
        }
        const int gi = lo, mi = mm - pp.pfx_offsets[gi];
        const int seq = pp.pfx_members[mm];
        if (mi >= pp.pfx_max_group || seq < 0 || seq >= ps.num_seqs)
            continue;                                 // flagged by the prefix pass
        int skipb = 0, e = 0;
        (void)stream_tokens(ps, seq, BS, capacity, skipb, e);
        if (skipb == 0)
            continue;                                 // nothing shared: the suffix pass wrote it whole
        // prefix pieces: stream (gi, h) of the prefix pass, column mi * Gq + gq (tile cg / 8)
        const int nb_p = (prefix_p[gi + 1] - prefix_p[gi]) / Hkv;
        const int pstream = gi * Hkv + h, sbp = prefix_p[gi] + h * nb_p;
        const int cg = mi * Gq + gq, tile = cg >> 3, c = cg & 7;
        const int fp = nb_p > 0 ? ch_p.of(sbp) : 0, np = nb_p > 0 ? ch_p.of(sbp + nb_p - 1) - fp + 1 : 0;
        // suffix pieces: stream (seq, h / HG) of the suffix pass, warp h % HG, column gq
        const int nb_s = (prefix_s[seq + 1] - prefix_s[seq]) / NHG;
        const int hg = h / HG, w = h - hg * HG, stream = seq * NHG + hg, sbs = prefix_s[seq] + hg * nb_s;
        const int fs = nb_s > 0 ? ch_s.of(sbs) : 0, ns = nb_s > 0 ? ch_s.of(sbs + nb_s - 1) - fs + 1 : 0;
        auto piece = [&](int i) -> PieceRef {
            if (i < np) {
                const float* b = pp.partials + ((size_t)(fp + i + pstream) * 4 + tile) * pp.slot_floats;
                return PieceRef{b + c * D, b + 8 * D + c, b + 8 * D + 8 + c};
            }
            const float* b = ps.partials + ((size_t)(fs + (i - np) + stream) * HG + w) * ps.slot_floats;
            return PieceRef{b + gq * D, b + G * D + gq, b + G * D + G + gq};
        };
        const float out_scale = ps.v_head_scales ? ps.v_scale * __ldg(ps.v_head_scales + h) : ps.v_scale;
        merge_column<QT, D>(np + ns, piece, out_scale,
                            reinterpret_cast<QT*>(ps.out) + ((size_t)seq * ps.num_heads + (size_t)h * Gq + gq) * D,
                            lane);
    }

    // (b) split streams of sequences without shared blocks
    const int items_b = ps.num_seqs * NHG * HG * G;
    for (int it = wid; it < items_b; it += warps) {
        const int gq = it % G, sw = it / G;
        const int stream = sw / HG, w = sw - stream * HG;
        const int s = stream / NHG, hg = stream - s * NHG;
        const int nb = (prefix_s[s + 1] - prefix_s[s]) / NHG;
        if (nb == 0)
            continue;
        int skipb = 0, e = 0;
        (void)stream_tokens(ps, s, BS, capacity, skipb, e);
        if (skipb > 0)
            continue;
        const int sb = prefix_s[s] + hg * nb;
        const int first_run = ch_s.of(sb), last_run = ch_s.of(sb + nb - 1);
        if (first_run != last_run)
            merge_split<QT, D, G, HG>(ps, s, stream, first_run, last_run - first_run + 1, NHG, w, gq, lane);
    }
}

// ------------------------------------------------------------------ host side

// Encode a 2-D tensor map over a cache: rows = num_blocks * num_kv_heads * block_size,
// row = head_dim elements, box = 128 bytes x box_rows, 128-byte swizzle.
bool make_cache_tensormap(CUtensorMap* map, const void* base, int kv_dtype, int head_dim, long long rows,
                          int box_rows);

// A merge kernel as a programmatic dependent launch behind the decode grid on `stream`.
inline int launch_merge_pdl(const void* kern, void** args, int grid, size_t smem, cudaStream_t stream)
{
    if (!ensure_smem_attribute(kern, smem))
        return PKV_ERR_LAUNCH;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kMergeThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelExC(&cfg, kern, args) == cudaSuccess ? PKV_OK : PKV_ERR_LAUNCH;
}

template <class KV, class QT, int D, int BS, int G, int HG, bool PFX = false>
struct MmaLauncher {
    using C = MmaCfg<KV, D, BS, G, HG, PFX>;

    static size_t smem_bytes(int num_seqs, int S)
    {
        return (size_t)S * C::kStage + (size_t)S * (8 + 8 + 4) + 16 + 2 * kChunkRing * 4 + (size_t)(num_seqs + 1) * 4 + 64;
    }

    // Ring depth: the SM's shared memory split between kCtasPerSM CTAs (~96 KB or ~64 KB of stages).
    static int stages(int num_seqs)
    {
        const long long budget = kMaxSmemPerBlock / C::kCtasPerSM - 1024;
        const long long room = budget - 16 - 2 * kChunkRing * 4 - (long long)(num_seqs + 1) * 4 - 64;
        long long S = room / (C::kStage + 20);
        if (S > 8)
            S = 8;
        if (S < 2) {   // many sequences: fall back to one CTA per SM
            S = ((long long)kMaxSmemPerBlock - 1024 - 16 - 2 * kChunkRing * 4 - (long long)(num_seqs + 1) * 4 - 64) /
                (C::kStage + 20);
            if (S > 8)
                S = 8;
        }
        return (int)S;
    }

    static int occupancy(int num_seqs)
    {
        const int S = stages(num_seqs);
        if (S < 2)
            return 0;
        auto kern = paged_decode_mma_kernel<KV, QT, D, BS, G, HG, PFX>;
        const size_t smem = smem_bytes(num_seqs, S);
        if (!ensure_smem_attribute((const void*)kern, smem))
            return 0;
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, C::kThreads, smem) != cudaSuccess)
            return 0;
        return n;
    }

    // The decode kernel alone (p gets the launcher's fields); `pdl`: as a programmatic dependent
    // launch behind the previous kernel on `stream`.
    static int launch_decode(DecodeParams& p, int nruns, cudaStream_t stream, bool pdl)
    {
        const int S = stages(p.num_seqs);
        if (S < 2)
            return PKV_ERR_SHAPE;
        const long long rows = (long long)p.num_blocks * p.num_kv_heads * BS;
        int kvdt = PKV_BF16;
        if constexpr (KV::kBytes == 1)
            kvdt = KV::kInt8 ? PKV_INT8 : KV::kFmt == __NV_E5M2 ? PKV_FP8_E5M2 : PKV_FP8_E4M3;
        CUtensorMap kmap, vmap;
        if (!make_cache_tensormap(&kmap, p.k_cache, kvdt, D, rows, C::kRows) ||
            !make_cache_tensormap(&vmap, p.v_cache, kvdt, D, rows, C::kRows))
            return PKV_ERR_LAUNCH;
        auto kern = paged_decode_mma_kernel<KV, QT, D, BS, G, HG, PFX>;
        const size_t smem = smem_bytes(p.num_seqs, S);
        if (!ensure_smem_attribute((const void*)kern, smem))
            return PKV_ERR_LAUNCH;
        p.stages_per_warp = S;
        // 8-bit codes enter the products widened exactly: only the per-tensor scales remain
        p.q_scale = p.scale * kLog2e * (KV::kBytes == 1 && !p.k_head_scales ? p.k_scale : 1.0f);
        p.v_scale = KV::kBytes == 1 && !p.v_head_scales ? p.v_scale_in : 1.0f;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(nruns);
        cfg.blockDim = dim3(C::kThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = pdl ? 1 : 0;
        return cudaLaunchKernelEx(&cfg, kern, kmap, vmap, p) == cudaSuccess ? PKV_OK : PKV_ERR_LAUNCH;
    }

    static int launch(DecodeParams p, int nruns, cudaStream_t stream)
    {
        const int st = launch_decode(p, nruns, stream, false);
        if (st != PKV_OK)
            return st;
        // the merge of split streams, allowed to start while the decode grid drains
        const int items = p.num_seqs * p.num_kv_heads * G;
        const int per_cta = kMergeThreads / 32;
        int mgrid = (items + per_cta - 1) / per_cta;
        if (mgrid > 2 * nruns)
            mgrid = 2 * nruns;
        void* args[] = {&p, &nruns};
        return launch_merge_pdl((const void*)paged_decode_merge_kernel<QT, D, BS, G, HG>, args, mgrid,
                                (size_t)(p.num_seqs + 1) * 4, stream);
    }

    // Shared-prefix decode: the prefix pass (pp: the plan's groups, one KV head per unit, 32 query
    // columns), then the suffix pass (ps: every sequence past its shared blocks) as a programmatic
    // dependent launch that may start while the prefix pass drains, then the merge of both.
    static int launch_shared_prefix(DecodeParams ps, DecodeParams pp, int runs_s, int runs_p, cudaStream_t stream)
    {
        using PL = MmaLauncher<KV, QT, D, BS, 8, 1, true>;
        const bool any_groups = pp.num_seqs > 0;
        if (any_groups) {
            const int st = PL::launch_decode(pp, runs_p, stream, false);
            if (st != PKV_OK)
                return st;
        }
        ps.wait_prior_at_exit = any_groups ? 1 : 0;
        const int st = launch_decode(ps, runs_s, stream, any_groups);
        if (st != PKV_OK)
            return st;
        const long long items = 1ll * ps.num_seqs * ps.num_kv_heads * G;   // >= members x query heads
        const int per_cta = kMergeThreads / 32;
        long long mgrid = (items + per_cta - 1) / per_cta;
        if (mgrid > 2ll * runs_s)
            mgrid = 2ll * runs_s;
        if (mgrid < 1)
            mgrid = 1;
        void* args[] = {&ps, &pp, &runs_s, &runs_p};
        return launch_merge_pdl((const void*)paged_decode_prefix_merge_kernel<QT, D, BS, G, HG>, args, (int)mgrid,
                                (size_t)(ps.num_seqs + 1 + pp.num_seqs + 1) * 4, stream);
    }
};

}  // namespace pkv
