// Paged decode attention for FP8 (E4M3 / E5M2) caches on the fifth-generation tensor cores of
// sm_100a: tcgen05.mma reads the 8-bit K and V tiles straight from the TMA stages in shared
// memory and accumulates in tensor memory (TMEM); no cache code is converted on the CUDA cores.
//
// Same result as the other decode kernels: for every sequence s and query head g,
// out[s][g] = softmax_t(scale * q . K_t) V_t over the seq_lens[s] cached tokens, K_t / V_t read
// through the block table ("vLLM inference cost optimisation", developer.aliyun.com, sections 2
// and 4; wzjinhao.cn vLLM write-up, section 2.1), GQA head g -> KV head g / Gq.
//
// Layout of the work:
//  * Unit = one cache block of a (sequence, head group) stream: the block's rows of HPU = 128 /
//    block_size consecutive KV heads, 128 rows of 128 bytes that lie contiguously in the cache
//    ([block][KV head][token][d]). One 2-D TMA box (128 rows, 128-byte swizzle) brings its K tile
//    and one its V tile: big copies, few of them (the TMA unit's cost is per copy). Units in
//    (sequence, head group, block) order are shared out in chunks as in the warp-MMA kernel
//    (Chunks); streams cut by a chunk boundary leave pieces for the merge.
//  * Tile row r = (head hl = r / block_size, token t = r % block_size). The scores are one
//    tcgen05.mma product S = K Q^T over all rows and all HPU heads' query columns (kind::f8f6f4,
//    M = 128 rows, N = the HPU heads x (E4M3 hi codes, lo codes) x G columns, padded so that each
//    softmax warp's heads start a 16-column group; four K = 32-byte steps of d); row r keeps only
//    its own head's columns. The weights go into P^T, where row
//    (head hl, column c) is non-zero only in the bytes of head hl's tokens, so O^T += V^T P^T
//    (M = 128 d, N = (head, column) pairs, K = 32 rows per step, P hi then P lo) sums each head's
//    own tokens only: the block-diagonal structure is exact, the extra tensor-core work is free.
//  * Warp 4 (producer): per unit, a table lookup (32 units resolved at once, one per lane, the
//    next 32 loaded while these are issued), the decode-step append of a stream's last block,
//    the unit's descriptor (sequence, head group, block, segment flags) and the two copies.
//  * Warp 5 issues the scores of every unit in order (once its tiles have landed and the S tile
//    has been read), warp 6 its p.V product (once the weights are in): a tcgen05.mma holds its
//    issuing thread for the tensor pipe's whole time (about 50 cycles for these shapes), so the
//    issuers are threads of their own, off the softmax warps' path.
//  * Warps 0-3 (softmax, 128 threads): thread i is TMEM lane i: tile row i for S (token t of head
//    hl), row d = i of O.
//  * One CTA per SM (the driver grants no more to a kernel that allocates tensor memory): the
//    SM's shared memory goes to a deep stage ring; the last quarter of the work is cut into small
//    chunks that CTAs claim as they run dry, so that slower SMs take fewer.
//  * q and p enter the 8-bit products as E4M3 hi + lo pairs: q scaled per column by a power of two
//    sigma (max |q| sigma < 256; a bf16 q is then held exactly down to 2^-2 of sigma's unit), p
//    times 2^6 under a lazy-max slack of 2 (so p 2^6 <= 256 and weights down to 2^-12 of the
//    running max stay E4M3-normal; the factor cancels between O and l).
//  * P tiles are double-buffered by unit parity; one S tile, one O tile (hi and lo parts) and one
//    Q tile, written at a segment's start (every score of the previous segment is done by then).
//  * Every wait is bounded; a wait that runs out sets PKV_DEVERR_TIMEOUT, every role leaves its
//    loop, thread 0 waits for the MMAs it issued, and TMEM is released before the CTA exits.
#pragma once

#include "decode_mma.cuh"

namespace pkv {

constexpr int kTcRows = 128;          // cache rows per unit (HPU heads x block_size tokens)
constexpr int kTcStage = 32768;       // K tile + V tile, 128 rows x 128 bytes each
constexpr int kTcThreads = 224;       // warps 0-3 softmax, 4 producer, 5 scores issuer, 6 p.V issuer

// ------------------------------------------------------------------ tcgen05 wrappers

// Shared-memory matrix descriptor (sm_100): start, leading / stride byte offsets (>> 4), the
// fixed version bits, 128-byte swizzle.
__device__ __forceinline__ uint64_t tc_sdesc(uint32_t saddr, uint32_t sbo)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;                         // leading byte offset (unused by swizzled layouts)
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;                         // 128-byte swizzle
    return d;
}

// Instruction descriptor of kind::f8f6f4: f32 accumulate, A / B formats (0 E4M3, 1 E5M2), A MN-major
// flag, N and M.
__device__ __forceinline__ constexpr uint32_t tc_idesc(uint32_t afmt, uint32_t bfmt, uint32_t a_mn, int N, int M)
{
    return (1u << 4) | (afmt << 7) | (bfmt << 10) | (a_mn << 15) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}

// Arrive on `bar` once every tcgen05.mma this thread issued before has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// TMEM loads / stores of this warp's 32 lanes, n consecutive 32-bit columns from `taddr`.
__device__ __forceinline__ void tc_ld16(uint32_t taddr, uint32_t* r)
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tc_ld8(uint32_t taddr, uint32_t* r)
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
}

__device__ __forceinline__ void tc_ld4(uint32_t taddr, uint32_t* r)
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr)
                 : "memory");
}

__device__ __forceinline__ void tc_ld2(uint32_t taddr, uint32_t* r)
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(taddr) : "memory");
}

__device__ __forceinline__ void tc_st16(uint32_t taddr, const uint32_t* r)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// n columns (a multiple of 2) in pieces of 16, 8, 4 and 2
template <int N>
__device__ __forceinline__ void tc_ld_cols(uint32_t taddr, uint32_t* r)
{
    static_assert(N % 2 == 0, "even column count");
    if constexpr (N >= 16) {
        tc_ld16(taddr, r);
        tc_ld_cols<N - 16>(taddr + 16, r + 16);
    } else if constexpr (N >= 8) {
        tc_ld8(taddr, r);
        tc_ld_cols<N - 8>(taddr + 8, r + 8);
    } else if constexpr (N >= 4) {
        tc_ld4(taddr, r);
        tc_ld_cols<N - 4>(taddr + 4, r + 4);
    } else if constexpr (N >= 2) {
        tc_ld2(taddr, r);
    }
}

// n columns, a multiple of 16
template <int N>
__device__ __forceinline__ void tc_st_cols(uint32_t taddr, const uint32_t* r)
{
    static_assert(N % 16 == 0, "multiple of 16 columns");
    if constexpr (N >= 16) {
        tc_st16(taddr, r);
        tc_st_cols<N - 16>(taddr + 16, r + 16);
    }
}

__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Two values (f16x2, low half first) as E4M3 hi and lo codes with hi + lo ~ x: hi = E4M3(x),
// lo = E4M3(x - hi), the difference exact in f16 (hi is x rounded to 4 significant bits). Each
// result holds its two codes in bits 0-15, the low half's first. |x| must stay below 448.
__device__ __forceinline__ void split_e4m3x2(uint32_t x, uint32_t& hi, uint32_t& lo)
{
    uint16_t h, l;
    uint32_t hv;
    asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;" : "=h"(h) : "r"(x));
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(hv) : "h"(h));
    const __half2 d = __hsub2(*reinterpret_cast<const __half2*>(&x), *reinterpret_cast<const __half2*>(&hv));
    asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;" : "=h"(l) : "r"(*reinterpret_cast<const uint32_t*>(&d)));
    hi = h;
    lo = l;
}

// Byte offset of byte b (0..127) of row r in a 128-byte-swizzled tile (1024-byte aligned).
__device__ __forceinline__ uint32_t swz_byte(int r, int b)
{
    return (uint32_t)(r * 128 + ((((b >> 4) ^ (r & 7)) << 4) | (b & 15)));
}


__device__ __forceinline__ void tc_st8(uint32_t taddr, const uint32_t* r)
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}

// TMEM loads / stores of n columns (a multiple of 8) in pieces of 8, from an 8-aligned column
template <int N>
__device__ __forceinline__ void tc_ld_cols8(uint32_t taddr, uint32_t* r)
{
    static_assert(N % 8 == 0, "multiple of 8 columns");
    if constexpr (N >= 8) {
        tc_ld8(taddr, r);
        tc_ld_cols8<N - 8>(taddr + 8, r + 8);
    }
}

template <int N>
__device__ __forceinline__ void tc_st_cols8(uint32_t taddr, const uint32_t* r)
{
    static_assert(N % 8 == 0, "multiple of 8 columns");
    if constexpr (N >= 8) {
        tc_st8(taddr, r);
        tc_st_cols8<N - 8>(taddr + 8, r + 8);
    }
}

// ------------------------------------------------------------------ configuration

template <class KV, class QT, int BS, int G>
struct TcCfg {
    static constexpr int HPU = kTcRows / BS;                  // KV heads per unit
    static constexpr int WH = 32 / BS;                        // heads per softmax warp
    static constexpr int NO = HPU * G;                        // (head, column) pairs of a unit
    static constexpr int NOp = (NO + 7) / 8 * 8;              // P^T rows per part = O columns per part
    static constexpr int kLdS = WH * 2 * G;                   // S columns of one softmax warp's heads
    static constexpr int kLdSp = (kLdS + 7) / 8 * 8;          // ... padded: each warp's columns start 8-aligned
    static constexpr int NQ = 4 * kLdSp;                      // Q^T rows = S columns per tile
    static constexpr int kTmemUsed = 2 * NQ + 2 * NOp;        // S0, S1, O (hi part, lo part)
    static constexpr int kTmemCols = kTmemUsed <= 32 ? 32 : kTmemUsed <= 64 ? 64 : kTmemUsed <= 128 ? 128
                                                          : kTmemUsed <= 256 ? 256 : 512;
    static constexpr int kQBytes = (NQ * 128 + 1023) / 1024 * 1024;
    static constexpr int kPBytes = 2 * NOp * 128;             // one buffer: hi rows, then lo rows
    // one CTA per SM (the occupancy the driver grants a kernel that allocates tensor memory)
    static constexpr int kCtasPerSm = 1;
    static constexpr uint32_t kFmt = KV::kFmt == __NV_E5M2 ? 1u : 0u;
    static_assert(KV::kBytes == 1 && !KV::kInt8, "FP8 caches");
    static_assert(BS == 16 || BS == 32, "block size");
    static_assert(G >= 1 && G <= 8, "query columns per KV head");
    static_assert(kTmemUsed <= 512 && NQ <= 256 && NQ % 16 == 0 && 2 * NOp <= 256, "tensor memory, MMA N");
    // Q^T row (= S column) of head hl of the unit, part 0 (hi codes) or 1 (lo codes), column c
    __device__ __forceinline__ static constexpr int qrow(int hl, int part, int c)
    {
        return (hl / WH) * kLdSp + (hl % WH) * 2 * G + part * G + c;
    }
};

// What the producer tells the softmax warps about the unit in a stage (written before the stage's
// full barrier is signalled).
struct TcDesc {
    int s, hg, j, flags;   // sequence, head group, block of the stream, kTc* flags
    int chunk, L, skip, pad;
};
constexpr int kTcFirst = 1;    // first unit of a segment (the units of one stream inside one chunk)
constexpr int kTcLast = 2;     // last unit of a segment
constexpr int kTcEnd = 4;      // no unit: the CTA's work is done
constexpr int kTcBad = 8;      // the block id was out of range: nothing was copied
constexpr int kTcDirect = 16;  // the stream lies in one chunk: output written directly

// ------------------------------------------------------------------ kernel

template <class KV, class QT, int BS, int G>
__global__ void __launch_bounds__(kTcThreads, (TcCfg<KV, QT, BS, G>::kCtasPerSm))
    paged_decode_tc05_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                             const DecodeParams p)
{
    using C = TcCfg<KV, QT, BS, G>;
    constexpr int D = 128;
    constexpr int HPU = C::HPU, NO = C::NO, NOp = C::NOp, NQ = C::NQ;
    constexpr float kSlack = 2.0f;     // log2 units
    constexpr float kPOff = 6.0f;      // p * 2^6 enters the products
    const int S = p.stages_per_warp;
    const int Hkv = p.num_kv_heads;
    const int NHG = Hkv / HPU;
    const int capacity = p.max_blocks_per_seq * BS;
    const int QL = p.q_len > 1 ? p.q_len : 1;
    const int Gq = p.num_heads / p.num_kv_heads;

    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* stages = smem;                                        // [S][32 KB]
    uint8_t* qtile = stages + (size_t)S * kTcStage;                // Q^T: NQ rows of 128 bytes
    uint8_t* ptile = qtile + C::kQBytes;                           // [2] P^T: NOp hi rows, NOp lo rows
    TcDesc* desc = reinterpret_cast<TcDesc*>(ptile + 2 * C::kPBytes);   // [S]
    uint64_t* bars = reinterpret_cast<uint64_t*>(desc + S);
    uint64_t* full = bars;                    // [S] the stage's copies have landed
    uint64_t* empty = full + S;               // [S] the stage's products are done
    uint64_t* s_full = empty + S;             // [2] the scores are in S tile b
    uint64_t* s_empty = s_full + 2;           // [2] every softmax warp has read S tile b
    uint64_t* p_full = s_empty + 2;           // [2] every softmax warp has written P
    uint64_t* p_empty = p_full + 2;           // [2] the p.V product reading P is done
    uint64_t* o_full = p_empty + 2;           // [1] the segment's last p.V is done
    uint64_t* o_empty = o_full + 1;           // [1] every softmax warp has read O
    uint64_t* q_full = o_empty + 1;           // [1] the segment's Q tile is written
    uint64_t* drain = q_full + 1;             // [2] each issuer's MMAs are done
    uint64_t* gbar = drain + 2;               // [1] the four softmax warps' group barrier
    int2* info = reinterpret_cast<int2*>(gbar + 1);                // [num_seqs] (tokens, skipped blocks)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(info + p.num_seqs);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* votes = reinterpret_cast<int*>(tmem_slot + 2);            // [2][4] lazy-max votes per warp
    float* colq = reinterpret_cast<float*>(votes + 8);             // [NO] score factor per (head, column)
    float* ash = colq + NO;                                        // [NO] rescale factors
    float* msh = ash + NO;                                         // [NO] running max at a segment's end
    float* lsh = msh + NO;                                         // [NO] weight sums at a segment's end
    int* prefix = reinterpret_cast<int*>(lsh + NO);                // [num_seqs + 1]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (tid == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_empty[i], 4);
            mbar_init(&p_full[i], 4);
            mbar_init(&p_empty[i], 1);
            mbar_init(&drain[i], 1);
        }
        mbar_init(o_full, 1);
        mbar_init(o_empty, 4);
        mbar_init(q_full, 1);
        mbar_init(gbar, 4);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                     "r"(C::kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // Q^T padding rows and the off-diagonal bytes of P^T are read by the tensor cores as zeros
    for (int i = tid; i < (C::kQBytes + 2 * C::kPBytes) / 16; i += kTcThreads)
        reinterpret_cast<uint4*>(qtile)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
    {
        const int bad = build_unit_prefix(p, prefix, BS, NHG, capacity, BS, info);   // ends with __syncthreads
        if (bad && blockIdx.x == 0 && tid == 0)
            atomicOr(p.err, bad);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int total = prefix[p.num_seqs];
    const int nruns = gridDim.x;
    const Chunks ch = make_chunks(total, nruns, p.tail_chunks, p.tail_min_units, p.tail_min_chunk);

    // zero rows of empty sequences (one run per sequence)
    for (int s = blockIdx.x; s < p.num_seqs; s += nruns) {
        if (prefix[s + 1] == prefix[s]) {
            if (tid == 0 && p.new_k != nullptr && __ldg(p.new_slots + s) >= 0)
                atomicOr(p.err, PKV_DEVERR_SLOT);
            if (info[s].y > 0)
                continue;
            const int rows = p.num_heads * QL;
            QT* o = reinterpret_cast<QT*>(p.out) + (size_t)s * rows * D;
            for (int i = tid; i < rows * D; i += kTcThreads)
                from_float(0.f, o + i);
        }
    }

    auto fail = [&]() {
        if (!*abort_flag) {
            *abort_flag = 1;
            atomicOr(p.err, PKV_DEVERR_TIMEOUT);
        }
    };

    if (warp == 4) {
        // =========================== producer ===============================
        // Units are resolved 32 at a time, one per lane; the next 32 table entries are loaded
        // while these units' copies are issued. Each stage gets the unit's descriptor.
        if (lane == 0) {
            prefetch_tensormap(&kmap);
            prefetch_tensormap(&vmap);
        }
        struct Look {
            int s, hg, j, nbl, phys, flags;
            bool has;
        };
        // unit x0 + lane of chunk [cb, ce): sequence, head group, block of the stream, blocks of the
        // stream, the raw table entry and the segment flags
        auto look = [&](int x0, int cb, int ce) -> Look {
            Look r{0, 0, 0, 0, 0, 0, false};
            const int x = x0 + lane;
            if (x < ce) {
                r.s = find_seq(prefix, p.num_seqs, x);
                const int nu = (prefix[r.s + 1] - prefix[r.s]) / NHG;
                const int rr = x - prefix[r.s];
                r.hg = rr / nu;
                r.j = rr - r.hg * nu;
                r.nbl = nu;
                r.has = true;
                const int skip = info[r.s].y;
                r.phys = __ldg(p.block_tables + (long long)r.s * p.max_blocks_per_seq + skip + r.j);
                const int sb = x - r.j;   // the stream's first unit
                r.flags = (x == cb || r.j == 0 ? kTcFirst : 0) | (x + 1 == ce || r.j == nu - 1 ? kTcLast : 0) |
                          (ch.of(sb) == ch.of(sb + nu - 1) && skip == 0 ? kTcDirect : 0);
            }
            return r;
        };
        int cur = blockIdx.x;
        bool aborted = false;
        int k = 0, issued = 0;
        while (cur < ch.C && !aborted) {
            const int cb = ch.begin(cur), ce = ch.end(cur);
            // The next chunk is claimed as this one's last unit is issued: the claim's round trip
            // overlaps the units still in the stages, and a CTA claims only once it is that far,
            // so the CTAs of slower SMs take fewer tail chunks.
            int nxt = ch.C;
            bool claimed = false;
            auto claim = [&]() {
                if (claimed)
                    return;
                claimed = true;
                if (ch.C > ch.R) {
                    int v = 0;
                    if (lane == 0)
                        v = ch.R + atomicAdd(p.chunk_ctr, 1);
                    nxt = __shfl_sync(kFullMask, v, 0);
                }
            };
            Look lk = look(cb, cb, ce);
            for (int x0 = cb; x0 < ce && !aborted; x0 += 32) {
                const Look nx = look(x0 + 32, cb, ce);   // loads in flight while this batch is issued
                const bool bad = lk.has && (lk.phys < 0 || lk.phys >= p.num_blocks);
                if (bad)
                    atomicOr(p.err, PKV_DEVERR_BLOCK_ID);
                // first cache row of the unit: block phys, KV head hg * HPU, token 0
                const int row = lk.has && !bad ? (lk.phys * Hkv + lk.hg * HPU) * BS : -1;
                const int nb = ce - x0 < 32 ? ce - x0 : 32;
                for (int q = 0; q < nb && !aborted; ++q, ++k) {
                    if (x0 + q == ce - 1)
                        claim();
                    const int sq = __shfl_sync(kFullMask, lk.s, q), hgq = __shfl_sync(kFullMask, lk.hg, q);
                    const int jq = __shfl_sync(kFullMask, lk.j, q), nblq = __shfl_sync(kFullMask, lk.nbl, q);
                    const int rowq = __shfl_sync(kFullMask, row, q), fq = __shfl_sync(kFullMask, lk.flags, q);
                    // the decode-step append of this stream's heads, before its last block is read
                    if (p.new_k != nullptr && jq == nblq - 1)
                        append_new_token_impl<KV>(p, sq, hgq * HPU, HPU, D, BS, lane, rowq < 0 ? -1 : rowq / (Hkv * BS));
                    if (lane == 0) {
                        const int st = k % S;
                        if (*abort_flag) {
                            aborted = true;
                        } else if (k >= S && !mbar_wait_bounded(&empty[st], ((k / S) - 1) & 1)) {
                            aborted = true;
                            fail();
                        } else if (p.withheld_unit != 0 && x0 + q == p.withheld_unit - 1) {
                            aborted = true;   // test hook: this stage never fills; issue nothing more
                        } else {
                            const int2 inf = info[sq];
                            reinterpret_cast<int4*>(desc + st)[0] = make_int4(sq, hgq, jq, fq | (rowq < 0 ? kTcBad : 0));
                            reinterpret_cast<int4*>(desc + st)[1] = make_int4(cur, inf.x, inf.y, 0);
                            if (rowq < 0) {
                                mbar_arrive(&full[st]);
                            } else {
                                mbar_arrive_expect_tx(&full[st], (uint32_t)kTcStage);
                                uint8_t* dst = stages + (size_t)st * kTcStage;
                                tma_load_2d(dst, &kmap, 0, rowq, &full[st]);
                                tma_load_2d(dst + kTcStage / 2, &vmap, 0, rowq, &full[st]);
                            }
                            issued = k + 1;
                        }
                    }
                    aborted = __shfl_sync(kFullMask, aborted ? 1 : 0, 0) != 0;
                }
                lk = nx;
            }
            if (!aborted)
                claim();   // an empty chunk
            cur = nxt;
        }
        // end of the work: a stage without bytes whose descriptor says so
        if (lane == 0 && !aborted) {
            const int st = k % S;
            if (k >= S && !mbar_wait_bounded(&empty[st], ((k / S) - 1) & 1)) {
                aborted = true;
                fail();
            } else {
                reinterpret_cast<int4*>(desc + st)[0] = make_int4(0, 0, 0, kTcEnd);
                mbar_arrive(&full[st]);
            }
        }
        if (lane == 0 && aborted) {
            for (int kk = max(0, issued - S); kk < issued; ++kk)
                (void)mbar_wait_bounded(&full[kk % S], (kk / S) & 1);
        }
    } else if (warp == 5) {
        // =========================== scores issuer ===========================
        // S = K Q^T of every unit in order into S tile k & 1: once its tiles have landed, the
        // softmax warps have read that tile (unit k - 2) and (a segment's first unit) the
        // segment's Q tile is written.
        if (lane == 0) {
            const uint32_t id_qk = tc_idesc(C::kFmt, 0u, 0u, NQ, 128);   // M 128 rows, N (head, hi/lo, column)
            const uint64_t q_desc = tc_sdesc(smem_addr(qtile), 1024);
            int seg = 0;
            bool ok = true;
            for (int k = 0; ok; ++k) {
                const int st = k % S;
                if (!mbar_wait_bounded(&full[st], (k / S) & 1)) {
                    ok = false;
                    break;
                }
                const int flags = reinterpret_cast<const int4*>(desc + st)[0].w;
                if (flags & kTcEnd)
                    break;
                if ((k >= 2 && !mbar_wait_bounded(&s_empty[k & 1], ((k >> 1) - 1) & 1)) ||
                    ((flags & kTcFirst) && !mbar_wait_bounded(q_full, seg & 1))) {
                    ok = false;
                    break;
                }
                if (flags & kTcFirst)
                    ++seg;
                tc_fence_after();
                const uint64_t k_desc = tc_sdesc(smem_addr(stages + (size_t)st * kTcStage), 1024);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)   // K steps of 32 bytes of d: start address + 32 bytes
                    tc_mma(tmem + (uint32_t)((k & 1) * NQ), k_desc + 2 * ks, q_desc + 2 * ks, id_qk, ks > 0 ? 1u : 0u);
                tc_commit(&s_full[k & 1]);
            }
            if (!ok)
                fail();
            tc_commit(&drain[0]);   // every MMA issued has completed before TMEM is released
            (void)mbar_wait_bounded(&drain[0], 0);
        }
        __syncwarp();
    } else if (warp == 6) {
        // =========================== p.V issuer ==============================
        // O^T += V^T [P_hi^T | P_lo^T] of every unit in order, once the softmax warps have written
        // its weights (a segment's first unit: once they have read the previous segment's O); its
        // completion frees the stage and the P buffer.
        if (lane == 0) {
            const uint32_t id_pv = tc_idesc(C::kFmt, 0u, 1u, 2 * NOp, 128);   // M 128 d (V^T MN-major)
            const uint32_t od = tmem + (uint32_t)(2 * NQ);
            int seg = 0;
            bool ok = true;
            for (int k = 0; ok; ++k) {
                const int st = k % S, b = k & 1;
                if (!mbar_wait_bounded(&full[st], (k / S) & 1)) {
                    ok = false;
                    break;
                }
                const int flags = reinterpret_cast<const int4*>(desc + st)[0].w;
                if (flags & kTcEnd)
                    break;
                const bool first = (flags & kTcFirst) != 0;
                if (!mbar_wait_bounded(&p_full[b], (k >> 1) & 1) ||
                    (first && seg >= 1 && !mbar_wait_bounded(o_empty, (seg - 1) & 1))) {
                    ok = false;
                    break;
                }
                if (first)
                    ++seg;
                tc_fence_after();
                const uint64_t v_desc = tc_sdesc(smem_addr(stages + (size_t)st * kTcStage + kTcStage / 2), 1024);
                const uint64_t p_desc = tc_sdesc(smem_addr(ptile + b * C::kPBytes), 1024);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)   // 32 tile rows per step: V + 4096 bytes, P + 32 bytes
                    tc_mma(od, v_desc + 256 * ks, p_desc + 2 * ks, id_pv, (first && ks == 0) ? 0u : 1u);
                tc_commit(&empty[st]);
                tc_commit(&p_empty[b]);
                if (flags & kTcLast)
                    tc_commit(o_full);
            }
            if (!ok)
                fail();
            tc_commit(&drain[1]);
            (void)mbar_wait_bounded(&drain[1], 0);
        }
        __syncwarp();
    } else {
        // =========================== softmax warps ===========================
        const int hl = tid / BS, t = tid - (tid / BS) * BS;            // this thread's tile row
        // this row's bytes of P^T (rows (hl, c), hi then lo; the byte is the tile row)
        uint32_t poh[G], pol[G];
#pragma unroll
        for (int c = 0; c < G; ++c) {
            poh[c] = swz_byte(hl * G + c, tid);
            pol[c] = swz_byte(NOp + hl * G + c, tid);
        }
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const uint32_t o_hi = tmem + (uint32_t)(2 * NQ) + lane_base, o_lo = o_hi + (uint32_t)NOp;   // row d = tid of O
        float m[G], lp[G], qk[G];
        int lim[G];
#pragma unroll
        for (int c = 0; c < G; ++c) {
            m[c] = -INFINITY;
            lp[c] = 0.f;
            qk[c] = 0.f;
            lim[c] = 0;
        }
        // Barrier of the four softmax warps with a bounded wait (an mbarrier, one arrival per warp;
        // a warp is never more than one phase ahead). No wait here can block for good: a warp
        // whose wait runs out leaves, and the others' waits run out in turn.
        uint32_t gphase = 0;
        auto group_sync = [&]() -> bool {
            __syncwarp();
            if (lane == 0)
                mbar_arrive(gbar);
            const bool okg = mbar_wait_bounded(gbar, gphase & 1);
            ++gphase;
            if (!okg)
                fail();
            return __all_sync(kFullMask, okg);
        };
        // Q^T of stream (s, hg): rows (head h2, hi / lo part, column c) at C::qrow, 16 threads per
        // (head, column) pair, 8 d each; colq = the pair's score factor (scale, log2 e, K scale,
        // 1 / sigma)
        auto write_q = [&](int s, int hg) {
            for (int task = tid; task < NO * 16; task += 128) {
                const int nn = task >> 4, d0 = (task & 15) * 8;
                const int h2 = nn / G, c = nn - (nn / G) * G;
                const int head = hg * HPU + h2;
                float f[8];
                load_q<8>(reinterpret_cast<const QT*>(p.q) + query_row(p, s, head, c) * D + d0, f);
                float mx = 0.f;
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    mx = fmaxf(mx, fabsf(f[i]));
#pragma unroll
                for (int off = 1; off < 16; off <<= 1)
                    mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, off));
                // mx < 2^(E - 126) with E its biased exponent; sigma = 2^(134 - E), kept normal both ways
                int se = 127;
                if (mx > 0.f) {
                    se = 127 + 134 - (int)((__float_as_uint(mx) >> 23) & 0xffu);
                    se = se < 2 ? 2 : (se > 252 ? 252 : se);
                }
                const float sig = __uint_as_float((uint32_t)se << 23);
                const float inv_sig = __uint_as_float((uint32_t)(254 - se) << 23);
                uint32_t hw[2], lw[2];
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    uint32_t h01, l01, h23, l23;
                    split_e4m3x2(pack2<true>(f[4 * i] * sig, f[4 * i + 1] * sig), h01, l01);
                    split_e4m3x2(pack2<true>(f[4 * i + 2] * sig, f[4 * i + 3] * sig), h23, l23);
                    hw[i] = h01 | (h23 << 16);
                    lw[i] = l01 | (l23 << 16);
                }
                *reinterpret_cast<uint2*>(qtile + swz_byte(C::qrow(h2, 0, c), d0)) = make_uint2(hw[0], hw[1]);
                *reinterpret_cast<uint2*>(qtile + swz_byte(C::qrow(h2, 1, c), d0)) = make_uint2(lw[0], lw[1]);
                if ((task & 15) == 0) {
                    const float hs = p.k_head_scales ? __ldg(p.k_head_scales + head) : 1.0f;
                    colq[nn] = p.q_scale * hs * inv_sig;
                }
            }
            fence_proxy_async_smem();   // read by the tensor cores once q_full is signalled
        };
        int nseg = 0;      // segments finished (O tile phases)
        // Two units per iteration (unit k and, when k is not the last of its segment, unit k + 1 of
        // the same stream): the syncs, fences and waits of an iteration are paid once for both.
        for (int k = 0;;) {
            const int st0 = k % S;
            if (!mbar_wait_bounded(&full[st0], (k / S) & 1)) {
                fail();
                break;
            }
            // the units (their stages' copies are done: the V rows below are read and written after them)
            const int4 da = reinterpret_cast<const int4*>(desc + st0)[0];
            const int4 db = reinterpret_cast<const int4*>(desc + st0)[1];
            const int flags = da.w;
            if (flags & kTcEnd)
                break;
            const int s = da.x, hg = da.y, chunk = db.x, L = db.y;
            const bool first = (flags & kTcFirst) != 0;
            const int nu = (flags & kTcLast) ? 1 : 2;   // units this iteration
            const int st1 = (k + 1) % S;
            int flags1 = kTcLast, j1 = 0;
            if (nu == 2) {
                if (!mbar_wait_bounded(&full[st1], ((k + 1) / S) & 1)) {
                    fail();
                    break;
                }
                const int4 d1 = reinterpret_cast<const int4*>(desc + st1)[0];
                flags1 = d1.w;
                j1 = d1.z;
            }
            const bool last = (flags1 & kTcLast) != 0;
            if (first) {
                // a new stream: its Q tile (the previous segment's scores are all done: their S tiles
                // were read) and the column factors and limits (column c: new token c / Gq of q_len)
                write_q(s, hg);
                if (!group_sync())
                    break;
                if (tid == 0)
                    mbar_arrive(q_full);
#pragma unroll
                for (int c = 0; c < G; ++c) {
                    qk[c] = colq[hl * G + c];
                    lim[c] = L - QL + 1 + c / Gq;
                    m[c] = -INFINITY;
                    lp[c] = 0.f;
                }
            }
            // ---- this row's scores in both units: the warp's heads' columns, then this head's hi and lo
            const int b0 = k & 1, b1 = (k + 1) & 1;
            if (!mbar_wait_bounded(&s_full[b0], (k >> 1) & 1) ||
                (nu == 2 && !mbar_wait_bounded(&s_full[b1], ((k + 1) >> 1) & 1))) {
                fail();
                break;
            }
            tc_fence_after();
            uint32_t r0[C::kLdSp], r1[C::kLdSp];
            tc_ld_cols8<C::kLdSp>(tmem + (uint32_t)(b0 * NQ + warp * C::kLdSp) + lane_base, r0);
            if (nu == 2)
                tc_ld_cols8<C::kLdSp>(tmem + (uint32_t)(b1 * NQ + warp * C::kLdSp) + lane_base, r1);
            tc_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&s_empty[b0]);
                if (nu == 2)
                    mbar_arrive(&s_empty[b1]);
            }
            const bool valid0 = da.z * BS + t < L && (flags & kTcBad) == 0;
            const bool valid1 = nu == 2 && j1 * BS + t < L && (flags1 & kTcBad) == 0;
            float sc0[G], sc1[G];
            bool exceed = false;
#pragma unroll
            for (int c = 0; c < G; ++c) {
                uint32_t h0 = r0[c], l0 = r0[G + c], h1 = r1[c], l1 = r1[G + c];
                if constexpr (C::WH == 2) {
                    if (lane >= 16) {
                        h0 = r0[2 * G + c];
                        l0 = r0[3 * G + c];
                        h1 = r1[2 * G + c];
                        l1 = r1[3 * G + c];
                    }
                }
                sc0[c] = (valid0 && da.z * BS + t < lim[c]) ? (__uint_as_float(h0) + __uint_as_float(l0)) * qk[c]
                                                            : -INFINITY;
                sc1[c] = (valid1 && j1 * BS + t < lim[c]) ? (__uint_as_float(h1) + __uint_as_float(l1)) * qk[c]
                                                          : -INFINITY;
                exceed |= fmaxf(sc0[c], sc1[c]) > m[c] + kSlack;
            }
            {
                const int vote = __any_sync(kFullMask, exceed);
                if (lane == 0)
                    votes[(gphase & 1) * 4 + warp] = vote;
            }
            const int vb = (gphase & 1) * 4;
            if (!group_sync())
                break;
            const int any = votes[vb] | votes[vb + 1] | votes[vb + 2] | votes[vb + 3];
            if (any) {
                // new reference per (head, column): the blocks' max where it passes the old one by
                // the slack (a head's tokens are lanes of one warp)
#pragma unroll
                for (int c = 0; c < G; ++c) {
                    float v = fmaxf(sc0[c], sc1[c]);
#pragma unroll
                    for (int off = BS / 2; off >= 1; off >>= 1)
                        v = fmaxf(v, __shfl_xor_sync(kFullMask, v, off));
                    float a = 1.f;
                    if (v > m[c] + kSlack) {
                        a = m[c] == -INFINITY ? 1.f : fast_exp2(m[c] - v);
                        m[c] = v;
                    }
                    lp[c] *= a;
                    if (t == 0)
                        ash[hl * G + c] = a;
                }
                if (!group_sync())
                    break;
                if (!first) {
                    // O holds the segment's earlier blocks: scale row d's columns once their p.V is done
                    const int kp = k - 1;
                    if (!mbar_wait_bounded(&p_empty[kp & 1], (kp >> 1) & 1)) {
                        fail();
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int c0 = 0; c0 < NOp; c0 += 8) {   // 8 columns of both parts at a time
                        uint32_t oh[8], ol[8];
                        tc_ld8(o_hi + c0, oh);
                        tc_ld8(o_lo + c0, ol);
                        tc_wait_ld();
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float a = c0 + i < NO ? ash[c0 + i] : 1.f;
                            oh[i] = __float_as_uint(__uint_as_float(oh[i]) * a);
                            ol[i] = __float_as_uint(__uint_as_float(ol[i]) * a);
                        }
                        tc_st8(o_hi + c0, oh);
                        tc_st8(o_lo + c0, ol);
                    }
                    tc_wait_st();
                }
            }
            // ---- weights, their hi / lo codes into P^T of each unit: row (head hl, column c),
            // byte = tile row; P buffer b was last read by the p.V of unit k - 2 (k - 1 for b1)
            float pr0[G], pr1[G];
#pragma unroll
            for (int c = 0; c < G; ++c) {
                pr0[c] = sc0[c] == -INFINITY ? 0.f : fast_exp2(sc0[c] - m[c] + kPOff);
                pr1[c] = sc1[c] == -INFINITY ? 0.f : fast_exp2(sc1[c] - m[c] + kPOff);
                lp[c] += pr0[c] + pr1[c];
            }
            if ((k >= 2 && !mbar_wait_bounded(&p_empty[b0], ((k >> 1) - 1) & 1)) ||
                (nu == 2 && k >= 1 && !mbar_wait_bounded(&p_empty[b1], (((k + 1) >> 1) - 1) & 1))) {
                fail();
                break;
            }
            uint8_t* pt0 = ptile + b0 * C::kPBytes;
            uint8_t* pt1 = ptile + b1 * C::kPBytes;
#pragma unroll
            for (int c = 0; c < G; c += 2) {
                uint32_t hi, lo;
                split_e4m3x2(pack2<true>(pr0[c], c + 1 < G ? pr0[c + 1] : 0.f), hi, lo);
                pt0[poh[c]] = (uint8_t)(hi & 0xff);
                pt0[pol[c]] = (uint8_t)(lo & 0xff);
                if (c + 1 < G) {
                    pt0[poh[c + 1]] = (uint8_t)(hi >> 8);
                    pt0[pol[c + 1]] = (uint8_t)(lo >> 8);
                }
                if (nu == 2) {
                    split_e4m3x2(pack2<true>(pr1[c], c + 1 < G ? pr1[c + 1] : 0.f), hi, lo);
                    pt1[poh[c]] = (uint8_t)(hi & 0xff);
                    pt1[pol[c]] = (uint8_t)(lo & 0xff);
                    if (c + 1 < G) {
                        pt1[poh[c + 1]] = (uint8_t)(hi >> 8);
                        pt1[pol[c + 1]] = (uint8_t)(lo >> 8);
                    }
                }
            }
            // weight 0 against V codes that may be NaN: zero this row of an invalid token's V tile
            if (!valid0) {
                uint4* vr = reinterpret_cast<uint4*>(stages + (size_t)st0 * kTcStage + kTcStage / 2 + tid * 128);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    vr[i] = make_uint4(0u, 0u, 0u, 0u);
            }
            if (nu == 2 && !valid1) {
                uint4* vr = reinterpret_cast<uint4*>(stages + (size_t)st1 * kTcStage + kTcStage / 2 + tid * 128);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    vr[i] = make_uint4(0u, 0u, 0u, 0u);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&p_full[b0]);
                if (nu == 2)
                    mbar_arrive(&p_full[b1]);
            }
            k += nu;
            if (!last)
                continue;

            // ---- end of the segment: its output
            if (!mbar_wait_bounded(o_full, nseg & 1)) {
                fail();
                break;
            }
            ++nseg;
            tc_fence_after();
            // l and the reference per (head, column) over the head's tokens
#pragma unroll
            for (int c = 0; c < G; ++c) {
                float v = lp[c];
#pragma unroll
                for (int off = BS / 2; off >= 1; off >>= 1)
                    v += __shfl_xor_sync(kFullMask, v, off);
                if (t == 0) {
                    lsh[hl * G + c] = v;
                    msh[hl * G + c] = m[c];
                }
            }
            if (!group_sync())
                break;
            const int stream = s * NHG + hg;
            const bool direct = (flags & kTcDirect) != 0;
#pragma unroll
            for (int c0 = 0; c0 < NOp; c0 += 8) {   // row d = tid of O, 8 columns of both parts at a time
                uint32_t oh[8], ol[8];
                tc_ld8(o_hi + c0, oh);
                tc_ld8(o_lo + c0, ol);
                tc_wait_ld();
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int nn = c0 + i;
                    if (nn >= NO)
                        continue;
                    const int h2 = nn / G, c2 = nn - (nn / G) * G, head = hg * HPU + h2;
                    const float o = __uint_as_float(oh[i]) + __uint_as_float(ol[i]);
                    if (direct) {   // thread tid writes element d = tid of every row
                        const float vs = p.v_head_scales ? p.v_scale * __ldg(p.v_head_scales + head) : p.v_scale;
                        const float l = lsh[nn];
                        from_float(o * (l > 0.f ? vs / l : 0.f),
                                   reinterpret_cast<QT*>(p.out) + query_row(p, s, head, c2) * D + tid);
                    } else {        // a piece per (chunk, stream, head): o, then m, then l
                        float* part = p.partials + ((size_t)(chunk + stream) * HPU + h2) * p.slot_floats;
                        part[c2 * D + tid] = o;
                        if (tid == nn) {
                            part[G * D + c2] = msh[nn] - kPOff;   // the reference the weights were taken against
                            part[G * D + G + c2] = lsh[nn];
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(o_empty);   // O has been read: the next segment's p.V may overwrite it
        }
    }

    // a suffix pass launched behind a prefix pass completes only after it
    if (p.wait_prior_at_exit && tid == 0)
        asm volatile("griddepcontrol.wait;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::kTmemCols)
                     : "memory");
}

// ------------------------------------------------------------------ host side

constexpr int kTcMaxStages = 8;
// Static split by default: tail chunks, claimed late (as a CTA issues its chunk's last unit),
// were measured at 8 to 16 units: each chunk is a new segment, and a segment boundary serialises
// this kernel's pipeline (the output, then the next Q tile, then the first scores), so the extra
// boundaries cost more than the per-SM imbalance they remove.
constexpr int kTcTailChunksPerRun = 0;
constexpr int kTcMinUnitsForTail = 32;
constexpr int kTcMinTailChunk = 16;

template <class KV, class QT, int BS, int G>
struct TcLauncher {
    using C = TcCfg<KV, QT, BS, G>;

    static size_t smem_bytes(int num_seqs, int S)
    {
        return (size_t)S * (kTcStage + sizeof(TcDesc) + 2 * 8) + C::kQBytes + 2 * C::kPBytes + 14 * 8 +
               (size_t)num_seqs * 8 + 8 + 8 * 4 + 4 * C::NO * 4 + (size_t)(num_seqs + 1) * 4 + 64;
    }

    // Ring depth: one CTA per SM, the SM's shared memory in stages
    static int stages(int num_seqs, int* ctas)
    {
        for (int S = kTcMaxStages; S >= 2; --S)
            if (smem_bytes(num_seqs, S) <= (size_t)kMaxSmemPerBlock - 1024) {
                *ctas = C::kCtasPerSm;
                return S;
            }
        *ctas = 0;
        return 0;
    }

    static int occupancy(int num_seqs)
    {
        int cps = 0;
        const int S = stages(num_seqs, &cps);
        if (S < 2)
            return 0;
        auto kern = paged_decode_tc05_kernel<KV, QT, BS, G>;
        const size_t smem = smem_bytes(num_seqs, S);
        if (!ensure_smem_attribute((const void*)kern, smem))
            return 0;
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kTcThreads, smem) != cudaSuccess)
            return 0;
        return n < cps ? n : cps;
    }

    static int launch(DecodeParams p, int nruns, cudaStream_t stream)
    {
        int cps = 0;
        const int S = stages(p.num_seqs, &cps);
        if (S < 2 || p.num_kv_heads % C::HPU != 0)
            return PKV_ERR_SHAPE;
        const long long rows = (long long)p.num_blocks * p.num_kv_heads * BS;
        const int kvdt = KV::kFmt == __NV_E5M2 ? PKV_FP8_E5M2 : PKV_FP8_E4M3;
        CUtensorMap kmap, vmap;
        if (!make_cache_tensormap(&kmap, p.k_cache, kvdt, 128, rows, kTcRows) ||
            !make_cache_tensormap(&vmap, p.v_cache, kvdt, 128, rows, kTcRows))
            return PKV_ERR_LAUNCH;
        auto kern = paged_decode_tc05_kernel<KV, QT, BS, G>;
        const size_t smem = smem_bytes(p.num_seqs, S);
        if (!ensure_smem_attribute((const void*)kern, smem))
            return PKV_ERR_LAUNCH;
        p.stages_per_warp = S;
        p.chunk_done = nullptr;   // this kernel does not stamp chunks: its merge waits for the grid
        // Units of 32 KB: up to kTcTailChunksPerRun tail chunks per CTA, from kTcMinUnitsForTail
        // units per CTA on, of kTcMinTailChunk units at least, claimed as CTAs run dry. A chunk
        // leaves pieces of HPU heads at slots (chunk + stream) * HPU + head: as many tail chunks
        // as the workspace's partial slots hold.
        const long long pairs = (long long)p.num_seqs * p.num_kv_heads;
        int tail = kTcTailChunksPerRun;
        while (tail > 0 && (long long)nruns * (1 + tail) * C::HPU + pairs > p.partial_slots)
            --tail;
        p.tail_chunks = tail;
        p.tail_min_units = kTcMinUnitsForTail;
        p.tail_min_chunk = kTcMinTailChunk;
        p.q_scale = p.scale * kLog2e * (!p.k_head_scales ? p.k_scale : 1.0f);
        p.v_scale = !p.v_head_scales ? p.v_scale_in : 1.0f;
        kern<<<nruns, kTcThreads, smem, stream>>>(kmap, vmap, p);
        if (cudaGetLastError() != cudaSuccess)
            return PKV_ERR_LAUNCH;
        // the merge of split streams (head groups of HPU KV heads, one block per unit)
        const int items = p.num_seqs * p.num_kv_heads * G;
        const int per_cta = kMergeThreads / 32;
        int mgrid = (items + per_cta - 1) / per_cta;
        if (mgrid > 2 * nruns)
            mgrid = 2 * nruns;
        void* args[] = {&p, &nruns};
        return launch_merge_pdl((const void*)paged_decode_merge_kernel<QT, 128, BS, G, C::HPU, BS>, args, mgrid,
                                (size_t)(p.num_seqs + 1) * 4, stream);
    }
};

}  // namespace pkv
