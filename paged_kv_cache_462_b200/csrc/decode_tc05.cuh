// Paged decode attention for FP8 (E4M3 / E5M2) caches on the fifth-generation tensor cores of
// sm_100a: tcgen05.mma reads the 8-bit K and V tiles straight from the TMA stages in shared
// memory and accumulates in tensor memory (TMEM); no cache code is converted on the CUDA cores.
//
// Same result as the other decode kernels: for every sequence s and query head g,
// out[s][g] = softmax_t(scale * q . K_t) V_t over the seq_lens[s] cached tokens, K_t / V_t read
// through the block table ("vLLM inference cost optimisation", developer.aliyun.com, sections 2
// and 4; wzjinhao.cn vLLM write-up, section 2.1), GQA head g -> KV head g / G.
//
// Layout of the work:
//  * Unit = 128 consecutive tokens (128 / block_size logical blocks) of one (sequence, KV head)
//    stream; units in (sequence, KV head, position) order are shared out in chunks exactly as in
//    the warp-MMA kernel (Chunks), and streams cut by a chunk boundary leave pieces for the merge.
//  * Warp 4 (producer): per unit, one 2-D TMA copy per block for K and one for V, each a box of
//    block_size rows x 128 bytes with 128-byte swizzle, landing at row (block index in the unit)
//    * block_size of the stage's 128-row K (V) tile, so a stage holds the unit as two
//    128 x 128-byte tiles in the layout the tensor cores read (K-major for K, MN-major for V).
//  * Warp 5 (MMA issuer, lane 0): S^T = K Q^T as four tcgen05.mma kind::f8f6f4 (M = 128 tokens,
//    N = 16: the 8 query columns as E4M3 hi codes, then the same 8 as lo codes, K = 32 bytes of d
//    each) into a TMEM S tile; when the softmax warps have written P, O^T += V^T P^T as eight
//    (M = 128 d, N = 8 columns, K = 32 tokens, P hi then P lo) into the stream's TMEM O tile.
//    Unit k+1's scores are issued before unit k's p.V, so the tensor cores work while the
//    softmax of unit k runs.
//  * Warps 0-3 (softmax, 128 threads): thread i is TMEM lane i, i.e. token i of the unit for S and
//    row d = i of O. It loads its token's 16 S values, forms the 8 columns' scaled scores, keeps
//    the online softmax (a lazy running max common to the 128 threads, partial sums per thread),
//    writes its token's weights as E4M3 hi and lo bytes into the P^T tile, and at the end of a
//    stream reads its row of O and writes the output row (or a partial piece).
//  * q and p enter the 8-bit products as E4M3 hi + lo pairs: q scaled per column by a power of two
//    sigma (max |q| sigma < 256; a bf16 q is then held exactly down to 2^-2 of sigma's unit), p
//    times 2^6 under a lazy-max slack of 2 (so p 2^6 <= 256 and weights down to 2^-12 of the
//    running max stay E4M3-normal; the factor cancels between O and l).
//  * S and P tiles are double-buffered by unit parity, Q and O tiles by stream (segment) parity.
//  * Every wait is bounded; a wait that runs out sets PKV_DEVERR_TIMEOUT, every role leaves its
//    loop, the MMA issuer drains its MMAs, and TMEM is released before the CTA exits.
#pragma once

#include "decode_mma.cuh"

namespace pkv {

constexpr int kTcUnit = 128;          // tokens per unit
constexpr int kTcStage = 32768;       // K tile + V tile, 128 rows x 128 bytes each
constexpr int kTcTmemCols = 64;       // S0 [0,16) S1 [16,32) O0 [32,40) O1 [40,48)
constexpr int kTcThreads = 192;       // warps 0-3 softmax, 4 producer, 5 MMA issuer

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

__device__ __forceinline__ void tc_ld16(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tc_ld8(uint32_t taddr, uint32_t (&r)[8])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
}

__device__ __forceinline__ void tc_st8(uint32_t taddr, const uint32_t (&r)[8])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
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

// ------------------------------------------------------------------ unit walk

// The CTA's units in order: chunk after chunk (ids from the producer's ring, read once the
// chunk's first stage has filled), units of a chunk in order, a segment = the units of one
// stream inside one chunk. Every role walks the same sequence.
struct TcUnit {
    int k;            // unit ordinal in the CTA (stage k % S, S/P buffer k & 1)
    int seg;          // segment ordinal in the CTA (Q/O buffer seg & 1)
    int chunk;        // chunk id
    int x;            // unit index
    int s, h;         // sequence, KV head
    int u;            // unit within the stream (tokens 128 u ..)
    int stream_begin, stream_end;
    bool first, last; // first / last unit of its segment
};

struct TcWalk {
    int ordinal;      // chunks consumed
    int chunk, x, end;
    int k, seg;
    bool done;

    __device__ __forceinline__ void init()
    {
        ordinal = 0;
        chunk = -1;
        x = end = 0;
        k = -1;
        seg = -1;
        done = false;
    }
};

// ------------------------------------------------------------------ kernel

template <class KV, class QT, int BS, int G>
struct TcCfg {
    static constexpr int kBPU = kTcUnit / BS;       // blocks per unit
    static constexpr uint32_t kFmt = KV::kFmt == __NV_E5M2 ? 1u : 0u;
    static_assert(KV::kBytes == 1 && !KV::kInt8, "FP8 caches");
    static_assert(BS == 16 || BS == 32, "block size");
    static_assert(G <= 8, "query columns per KV head");
};

template <class KV, class QT, int BS, int G>
__global__ void __launch_bounds__(kTcThreads, 2)
    paged_decode_tc05_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                             const DecodeParams p)
{
    using C = TcCfg<KV, QT, BS, G>;
    constexpr int D = 128;
    constexpr float kSlack = 2.0f;     // log2 units
    constexpr float kPOff = 6.0f;      // p * 2^6 enters the products
    const int S = p.stages_per_warp;
    const int Hkv = p.num_kv_heads;
    const int capacity = p.max_blocks_per_seq * BS;
    const int QL = p.q_len > 1 ? p.q_len : 1;
    const int Gq = p.num_heads / p.num_kv_heads;

    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* stages = smem;                                        // [S][32 KB]
    uint8_t* qtile = stages + (size_t)S * kTcStage;                // [2][2 KB]
    uint8_t* ptile = qtile + 2 * 2048;                             // [2][2 KB]
    uint64_t* bars = reinterpret_cast<uint64_t*>(ptile + 2 * 2048);
    uint64_t* full = bars;                    // [S]
    uint64_t* empty = full + S;               // [S]
    uint64_t* s_full = empty + S;             // [2]
    uint64_t* s_empty = s_full + 2;           // [2]
    uint64_t* p_full = s_empty + 2;           // [2]
    uint64_t* p_empty = p_full + 2;           // [2]
    uint64_t* o_full = p_empty + 2;           // [2]
    uint64_t* o_empty = o_full + 2;           // [2]
    uint64_t* q_full = o_empty + 2;           // [2]
    uint64_t* q_empty = q_full + 2;           // [2]
    uint64_t* drain = q_empty + 2;            // [1]
    uint64_t* gbar = drain + 1;               // [1] the four softmax warps' group barrier
    int* stage_bad = reinterpret_cast<int*>(gbar + 1);             // [S] bad-block bit masks
    int* chunk_ring = stage_bad + S;                               // [kChunkRing]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(chunk_ring + kChunkRing);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* red = reinterpret_cast<float*>(tmem_slot + 2);          // [4][8] cross-warp reductions
    float* colq = red + 32;                                        // [2][8] per-column score factors
    int* votes = reinterpret_cast<int*>(colq + 16);                // [2][4] lazy-max votes per warp
    int* prefix = votes + 8;                                       // [num_seqs + 1]

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
            mbar_init(&o_full[i], 1);
            mbar_init(&o_empty[i], 4);
            mbar_init(&q_full[i], 4);
            mbar_init(&q_empty[i], 1);
        }
        mbar_init(drain, 1);
        mbar_init(gbar, 4);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                     "r"(kTcTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // tiles read by the tensor cores start as zeros (rows no copy fills must not hold NaN codes)
    for (int i = tid; i < (S * kTcStage + 4 * 2048) / 16; i += kTcThreads)
        reinterpret_cast<uint4*>(stages)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
    {
        const int bad = build_unit_prefix(p, prefix, BS, Hkv, capacity, kTcUnit);   // ends with __syncthreads
        if (bad && blockIdx.x == 0 && tid == 0)
            atomicOr(p.err, bad);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int total = prefix[p.num_seqs];
    const int nruns = gridDim.x;
    const Chunks ch = make_chunks(total, nruns, p.tail_chunks);

    // zero rows of empty sequences (one run per sequence)
    for (int s = blockIdx.x; s < p.num_seqs; s += nruns) {
        if (prefix[s + 1] == prefix[s]) {
            if (tid == 0 && p.new_k != nullptr && __ldg(p.new_slots + s) >= 0)
                atomicOr(p.err, PKV_DEVERR_SLOT);
            if (p.skip_blocks != nullptr) {
                int skipb, e = 0;
                (void)stream_tokens(p, s, BS, capacity, skipb, e);
                if (skipb > 0)
                    continue;
            }
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
    // next unit of the walk (false at the end of the CTA's work or on a failed wait); a chunk's
    // id is read once the chunk's first stage has filled
    auto next_unit = [&](TcWalk& w, TcUnit& u) -> bool {
        if (w.done)
            return false;
        if (w.x >= w.end) {
            const int kk = w.k + 1;
            if (*abort_flag || !mbar_wait_bounded(&full[kk % S], (kk / S) & 1)) {
                fail();
                w.done = true;
                return false;
            }
            const int c = chunk_ring[w.ordinal % kChunkRing];
            ++w.ordinal;
            if (c < 0 || c >= ch.C) {
                w.done = true;
                return false;
            }
            w.chunk = c;
            w.x = ch.begin(c);
            w.end = ch.end(c);
        }
        u.k = ++w.k;
        u.chunk = w.chunk;
        u.x = w.x;
        u.s = find_seq(prefix, p.num_seqs, w.x);
        const int nu = (prefix[u.s + 1] - prefix[u.s]) / Hkv;
        const int r = w.x - prefix[u.s];
        u.h = r / nu;
        u.u = r - u.h * nu;
        u.stream_begin = prefix[u.s] + u.h * nu;
        u.stream_end = u.stream_begin + nu;
        u.first = w.x == ch.begin(w.chunk) || w.x == u.stream_begin;
        u.last = w.x + 1 == w.end || w.x + 1 == u.stream_end;
        if (u.first)
            ++w.seg;
        u.seg = w.seg;
        ++w.x;
        return true;
    };

    if (warp == 4) {
        // =========================== producer ===============================
        if (lane == 0) {
            prefetch_tensormap(&kmap);
            prefetch_tensormap(&vmap);
        }
        int cur = blockIdx.x;
        int nxt = ch.C;
        if (lane == 0 && ch.C > ch.R)
            nxt = ch.R + atomicAdd(p.chunk_ctr, 1);
        bool aborted = false;
        int k = 0, issued = 0, published = 0;
        while (cur < ch.C && !aborted) {
            const int cb = ch.begin(cur), ce = ch.end(cur);
            if (ce > cb) {
                if (lane == 0)
                    chunk_ring[published % kChunkRing] = cur;
                ++published;
            }
            for (int x = cb; x < ce && !aborted; ++x, ++k) {
                const int s = find_seq(prefix, p.num_seqs, x);
                const int nu = (prefix[s + 1] - prefix[s]) / Hkv;
                const int r = x - prefix[s];
                const int h = r / nu, uu = r - h * nu;
                int skipb = 0, L = 0;
                {
                    int e = 0;
                    L = stream_tokens(p, s, BS, capacity, skipb, e);
                }
                const int nbl = (L + BS - 1) / BS;               // blocks of the stream
                const int j0 = uu * C::kBPU;
                // lane b < kBPU: block j0 + b of the stream -> pool row, -1 when past the stream or bad
                int row = -1, bad = 0;
                if (lane < C::kBPU && j0 + lane < nbl) {
                    const int phys = __ldg(p.block_tables + (long long)s * p.max_blocks_per_seq + skipb + j0 + lane);
                    if (phys < 0 || phys >= p.num_blocks) {
                        atomicOr(p.err, PKV_DEVERR_BLOCK_ID);
                        bad = 1;
                    } else {
                        row = (phys * Hkv + h) * BS;
                    }
                }
                const unsigned badmask = __ballot_sync(kFullMask, bad != 0);
                const unsigned loadmask = __ballot_sync(kFullMask, row >= 0);
                // the decode-step append of this stream, before its last block is read
                if (p.new_k != nullptr && j0 + C::kBPU >= nbl && nbl > 0) {
                    const int lastrow = __shfl_sync(kFullMask, row, (nbl - 1 - j0) & 31);
                    append_new_token_impl<KV>(p, s, h, 1, D, BS, lane, lastrow < 0 ? -1 : lastrow / (Hkv * BS));
                }
                if (lane == 0) {
                    const int st = k % S;
                    if (*abort_flag) {
                        aborted = true;
                    } else if (k >= S && !mbar_wait_bounded(&empty[st], ((k / S) - 1) & 1)) {
                        aborted = true;
                        fail();
                    } else if (p.withheld_unit != 0 && x == p.withheld_unit - 1) {
                        aborted = true;   // test hook: this stage never fills; issue nothing more
                    } else {
                        stage_bad[st] = (int)badmask;
                        const int n = __popc(loadmask);
                        if (n == 0)
                            mbar_arrive(&full[st]);
                        else
                            mbar_arrive_expect_tx(&full[st], (uint32_t)n * BS * 128 * 2);
                        issued = k + 1;
                    }
                }
                // the copies (lane 0 issues; rows broadcast from the lanes that resolved them)
                const int st = k % S;
                const bool go = __shfl_sync(kFullMask, (int)(!aborted && issued == k + 1), 0) != 0;
                aborted = __shfl_sync(kFullMask, aborted ? 1 : 0, 0) != 0;
#pragma unroll
                for (int b = 0; b < C::kBPU; ++b) {
                    const int rb = __shfl_sync(kFullMask, row, b);
                    if (go && lane == 0 && rb >= 0) {
                        uint8_t* dst = stages + (size_t)st * kTcStage + b * BS * 128;
                        tma_load_2d(dst, &kmap, 0, rb, &full[st]);
                        tma_load_2d(dst + kTcStage / 2, &vmap, 0, rb, &full[st]);
                    }
                }
            }
            cur = __shfl_sync(kFullMask, nxt, 0);
            if (lane == 0 && cur < ch.C)
                nxt = ch.R + atomicAdd(p.chunk_ctr, 1);
        }
        // end of the work: a stage without bytes whose chunk id is -1 tells the other roles
        if (lane == 0 && !aborted) {
            const int st = k % S;
            if (k >= S && !mbar_wait_bounded(&empty[st], ((k / S) - 1) & 1)) {
                aborted = true;
                fail();
            } else {
                chunk_ring[published % kChunkRing] = -1;
                stage_bad[st] = 0;
                mbar_arrive(&full[st]);
            }
        }
        if (lane == 0 && aborted) {
            for (int kk = max(0, issued - S); kk < issued; ++kk)
                (void)mbar_wait_bounded(&full[kk % S], (kk / S) & 1);
        }
    } else if (warp == 5) {
        // =========================== MMA issuer ==============================
        if (lane == 0) {
            const uint32_t id_qk = tc_idesc(C::kFmt, 0u, 0u, 16, 128);
            const uint32_t id_pv = tc_idesc(C::kFmt, 0u, 1u, 8, 128);
            TcWalk wq, wp;
            wq.init();
            wp.init();
            TcUnit uq, up;
            auto issue_qk = [&](const TcUnit& u) -> bool {
                const int st = u.k % S, b = u.k & 1, n = u.k >> 1, j = u.seg & 1;
                // next_unit already waited for the first stage of a chunk; wait for this one
                if (!mbar_wait_bounded(&full[st], (u.k / S) & 1))
                    return false;
                if (n >= 1 && !mbar_wait_bounded(&s_empty[b], (n - 1) & 1))
                    return false;
                if (u.first && !mbar_wait_bounded(&q_full[j], (u.seg >> 1) & 1))
                    return false;
                tc_fence_after();
                const uint32_t kbase = smem_addr(stages + (size_t)st * kTcStage);
                const uint32_t qbase = smem_addr(qtile + j * 2048);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc_mma(tmem + 16u * b, tc_sdesc(kbase + ks * 32, 1024), tc_sdesc(qbase + ks * 32, 1024), id_qk,
                           ks > 0 ? 1u : 0u);
                tc_commit(&s_full[b]);
                if (u.last)
                    tc_commit(&q_empty[j]);
                return true;
            };
            bool ok = true;
            bool have_q = next_unit(wq, uq);
            if (have_q)
                ok = issue_qk(uq);
            while (ok && next_unit(wp, up)) {
                if (next_unit(wq, uq))
                    ok = issue_qk(uq);
                if (!ok)
                    break;
                const int st = up.k % S, b = up.k & 1, n = up.k >> 1, j = up.seg & 1;
                if (!mbar_wait_bounded(&p_full[b], n & 1)) {
                    ok = false;
                    break;
                }
                if (up.first && up.seg >= 2 && !mbar_wait_bounded(&o_empty[j], ((up.seg >> 1) - 1) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t vbase = smem_addr(stages + (size_t)st * kTcStage + kTcStage / 2);
                const uint32_t pbase = smem_addr(ptile + b * 2048);
                const uint32_t od = tmem + 32u + 8u * j;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t a = tc_sdesc(vbase + ks * 4096, 1024);
                    tc_mma(od, a, tc_sdesc(pbase + ks * 32, 1024), id_pv, (up.first && ks == 0) ? 0u : 1u);
                    tc_mma(od, a, tc_sdesc(pbase + 1024 + ks * 32, 1024), id_pv, 1u);
                }
                tc_commit(&empty[st]);
                tc_commit(&p_empty[b]);
                if (up.last)
                    tc_commit(&o_full[j]);
            }
            if (!ok)
                fail();
            // every MMA issued has completed before TMEM is released
            tc_commit(drain);
            (void)mbar_wait_bounded(drain, 0);
        }
        __syncwarp();
    } else {
        // =========================== softmax warps ===========================
        const float qk_head_scale = p.q_scale;   // per-tensor factor (head scales applied per stream)
        TcWalk w;
        w.init();
        TcUnit u;
        float m[8], lp[8], qk[8];
        int lim[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            m[c] = -INFINITY;
            lp[c] = 0.f;
            qk[c] = 0.f;
            lim[c] = 0;
        }
        int q_written = -1;   // last segment whose Q tile is written
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
        // Q tile of segment u.seg: thread i -> column i >> 4, d (i & 15) * 8 .. + 7
        auto write_q = [&](const TcUnit& uu) -> bool {
            const int j = uu.seg & 1;
            if (uu.seg >= 2 && !mbar_wait_bounded(&q_empty[j], ((uu.seg >> 1) - 1) & 1))
                return false;
            const int c = tid >> 4, d0 = (tid & 15) * 8;
            float f[8];
            if (c < G) {
                const QT* qp = reinterpret_cast<const QT*>(p.q) + query_row(p, uu.s, uu.h, c) * D + d0;
                load_q<8>(qp, f);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    f[i] = 0.f;
            }
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
            uint8_t* qt = qtile + j * 2048;
            *reinterpret_cast<uint2*>(qt + swz_byte(c, d0)) = make_uint2(hw[0], hw[1]);
            *reinterpret_cast<uint2*>(qt + swz_byte(8 + c, d0)) = make_uint2(lw[0], lw[1]);
            const float hs = p.k_head_scales ? __ldg(p.k_head_scales + uu.h) : 1.0f;
            if ((tid & 15) == 0)
                colq[j * 8 + c] = qk_head_scale * hs * inv_sig;
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&q_full[j]);
            return true;
        };
        bool ok = next_unit(w, u);
        if (ok)
            ok = write_q(u);
        if (ok)
            q_written = u.seg;
        while (ok) {
            const int st = u.k % S, b = u.k & 1, n = u.k >> 1, j = u.seg & 1;
            int skipb = 0, L = 0;
            {
                int e = 0;
                L = stream_tokens(p, u.s, BS, capacity, skipb, e);
            }
            if (u.first) {
                // the segment's column factors and limits (column c: new token c / Gq of q_len)
                if (!group_sync())   // colq of this segment written by write_q
                    break;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    qk[c] = colq[j * 8 + c];
                    lim[c] = c < G ? L - QL + 1 + c / Gq : 0;
                    m[c] = -INFINITY;
                    lp[c] = 0.f;
                }
            }
            // ---- scores of token tid of this unit (the stage's copies are done: stage_bad and the V
            // rows below are read and written after them)
            if (!mbar_wait_bounded(&full[st], (u.k / S) & 1) || !mbar_wait_bounded(&s_full[b], n & 1)) {
                fail();
                break;
            }
            tc_fence_after();
            uint32_t r[16];
            tc_ld16(tmem + 16u * b + ((uint32_t)(warp * 32) << 16), r);
            tc_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&s_empty[b]);
            const int pos = u.u * kTcUnit + tid;
            const bool valid = pos < L && !((stage_bad[st] >> (tid / BS)) & 1);
            float sc[8];
            bool exceed = false;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float raw = __uint_as_float(r[c]) + __uint_as_float(r[8 + c]);
                sc[c] = (valid && pos < lim[c]) ? raw * qk[c] : -INFINITY;
                exceed |= sc[c] > m[c] + kSlack;
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
                // new reference: the 128 tokens' max per column where it passes the old one by the slack
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    float v = sc[c];
#pragma unroll
                    for (int off = 16; off >= 1; off >>= 1)
                        v = fmaxf(v, __shfl_xor_sync(kFullMask, v, off));
                    if (lane == 0)
                        red[warp * 8 + c] = v;
                }
                if (!group_sync())
                    break;
                float a[8];
                bool rescale = false;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float M = fmaxf(fmaxf(red[c], red[8 + c]), fmaxf(red[16 + c], red[24 + c]));
                    a[c] = 1.f;
                    if (M > m[c] + kSlack) {
                        a[c] = m[c] == -INFINITY ? 1.f : fast_exp2(m[c] - M);
                        rescale |= m[c] != -INFINITY;
                        m[c] = M;
                    }
                    lp[c] *= a[c];
                }
                if (!group_sync())   // red reused later
                    break;
                if (rescale && !u.first) {
                    // O holds the segment's earlier units: scale it once their p.V products are done
                    const int kp = u.k - 1;
                    if (!mbar_wait_bounded(&p_empty[kp & 1], (kp >> 1) & 1)) {
                        fail();
                        break;
                    }
                    tc_fence_after();
                    uint32_t o[8];
                    const uint32_t ot = tmem + 32u + 8u * j + ((uint32_t)(warp * 32) << 16);
                    tc_ld8(ot, o);
                    tc_wait_ld();
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        o[c] = __float_as_uint(__uint_as_float(o[c]) * a[c]);
                    tc_st8(ot, o);
                    tc_wait_st();
                }
            }
            // ---- weights, their hi / lo codes into P^T (row c hi, row 8 + c lo; byte = token)
            float pr[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                pr[c] = sc[c] == -INFINITY ? 0.f : fast_exp2(sc[c] - m[c] + kPOff);
                lp[c] += pr[c];
            }
            if (n >= 1 && !mbar_wait_bounded(&p_empty[b], (n - 1) & 1)) {
                fail();
                break;
            }
            uint8_t* pt = ptile + b * 2048;
#pragma unroll
            for (int c = 0; c < 8; c += 2) {
                uint32_t hi, lo;
                split_e4m3x2(pack2<true>(pr[c], pr[c + 1]), hi, lo);
                pt[swz_byte(c, tid)] = (uint8_t)(hi & 0xff);
                pt[swz_byte(c + 1, tid)] = (uint8_t)(hi >> 8);
                pt[swz_byte(8 + c, tid)] = (uint8_t)(lo & 0xff);
                pt[swz_byte(9 + c, tid)] = (uint8_t)(lo >> 8);
            }
            if (!valid) {   // weight 0 against V codes that may be NaN: zero this token's V row
                uint4* vr = reinterpret_cast<uint4*>(stages + (size_t)st * kTcStage + kTcStage / 2 + tid * 128);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    vr[i] = make_uint4(0u, 0u, 0u, 0u);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&p_full[b]);

            if (!u.last) {
                ok = next_unit(w, u);
                continue;
            }
            // ---- end of the segment: next segment's Q first (the tensor cores can start on it),
            // then this segment's output
            const TcUnit cur = u;
            const int curL = L;
            bool more = next_unit(w, u);
            if (more) {
                if (!write_q(u)) {
                    fail();
                    more = false;
                } else {
                    q_written = u.seg;
                }
            }
            if (!mbar_wait_bounded(&o_full[j], (cur.seg >> 1) & 1)) {
                fail();
                break;
            }
            tc_fence_after();
            uint32_t o[8];
            tc_ld8(tmem + 32u + 8u * j + ((uint32_t)(warp * 32) << 16), o);
            tc_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&o_empty[j]);
            // l per column over the 128 tokens
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                float v = lp[c];
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1)
                    v += __shfl_xor_sync(kFullMask, v, off);
                if (lane == 0)
                    red[warp * 8 + c] = v;
            }
            if (!group_sync())
                break;
            float lsum[8];
#pragma unroll
            for (int c = 0; c < 8; ++c)
                lsum[c] = red[c] + red[8 + c] + red[16 + c] + red[24 + c];
            if (!group_sync())
                break;
            const float vs = p.v_head_scales ? p.v_scale * __ldg(p.v_head_scales + cur.h) : p.v_scale;
            const int stream = cur.s * Hkv + cur.h;
            const int first_chunk = ch.of(cur.stream_begin), last_chunk = ch.of(cur.stream_end - 1);
            if (first_chunk == last_chunk && skipb == 0) {
#pragma unroll
                for (int c = 0; c < G; ++c) {
                    const float inv = lsum[c] > 0.f ? vs / lsum[c] : 0.f;
                    QT* dst = reinterpret_cast<QT*>(p.out) + query_row(p, cur.s, cur.h, c) * D + tid;
                    from_float(__uint_as_float(o[c]) * inv, dst);
                }
            } else {
                float* part = p.partials + (size_t)(cur.chunk + stream) * p.slot_floats;
#pragma unroll
                for (int c = 0; c < G; ++c)
                    part[c * D + tid] = __uint_as_float(o[c]);
#pragma unroll
                for (int c = 0; c < G; ++c)
                    if (tid == c) {
                        part[G * D + c] = m[c] - kPOff;   // the reference the weights were taken against
                        part[G * D + G + c] = lsum[c];
                    }
            }
            (void)curL;
            ok = more;
        }
        (void)q_written;
    }

    // a suffix pass launched behind a prefix pass completes only after it
    if (p.wait_prior_at_exit && tid == 0)
        asm volatile("griddepcontrol.wait;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcTmemCols)
                     : "memory");
}

// ------------------------------------------------------------------ host side

template <class KV, class QT, int BS, int G>
struct TcLauncher {
    static size_t smem_bytes(int num_seqs, int S)
    {
        return (size_t)S * kTcStage + 4 * 2048 + (size_t)(2 * S + 18) * 8 + (size_t)S * 4 + kChunkRing * 4 + 8 +
               (32 + 16 + 8) * 4 + (size_t)(num_seqs + 1) * 4 + 64;
    }

    // Ring depth: two CTAs per SM, the rest of the SM's shared memory in stages
    static int stages(int num_seqs)
    {
        for (int S = 3; S >= 2; --S)
            if (smem_bytes(num_seqs, S) + 1024 <= (size_t)kMaxSmemPerBlock / 2)
                return S;
        for (int S = 4; S >= 2; --S)   // many sequences: one CTA per SM
            if (smem_bytes(num_seqs, S) + 1024 <= (size_t)kMaxSmemPerBlock)
                return S;
        return 0;
    }

    static int occupancy(int num_seqs)
    {
        const int S = stages(num_seqs);
        if (S < 2)
            return 0;
        auto kern = paged_decode_tc05_kernel<KV, QT, BS, G>;
        const size_t smem = smem_bytes(num_seqs, S);
        if (!ensure_smem_attribute((const void*)kern, smem))
            return 0;
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kTcThreads, smem) != cudaSuccess)
            return 0;
        return n < 2 ? n : 2;   // 2 x 64 TMEM columns per SM at most is what the kernel plans for
    }

    static int launch(DecodeParams p, int nruns, cudaStream_t stream)
    {
        const int S = stages(p.num_seqs);
        if (S < 2)
            return PKV_ERR_SHAPE;
        const long long rows = (long long)p.num_blocks * p.num_kv_heads * BS;
        const int kvdt = KV::kFmt == __NV_E5M2 ? PKV_FP8_E5M2 : PKV_FP8_E4M3;
        CUtensorMap kmap, vmap;
        if (!make_cache_tensormap(&kmap, p.k_cache, kvdt, 128, rows, BS) ||
            !make_cache_tensormap(&vmap, p.v_cache, kvdt, 128, rows, BS))
            return PKV_ERR_LAUNCH;
        auto kern = paged_decode_tc05_kernel<KV, QT, BS, G>;
        const size_t smem = smem_bytes(p.num_seqs, S);
        if (!ensure_smem_attribute((const void*)kern, smem))
            return PKV_ERR_LAUNCH;
        p.stages_per_warp = S;
        p.q_scale = p.scale * kLog2e * (!p.k_head_scales ? p.k_scale : 1.0f);
        p.v_scale = !p.v_head_scales ? p.v_scale_in : 1.0f;
        kern<<<nruns, kTcThreads, smem, stream>>>(kmap, vmap, p);
        if (cudaGetLastError() != cudaSuccess)
            return PKV_ERR_LAUNCH;
        // the merge of split streams (one KV head per stream, 128-token units)
        const int items = p.num_seqs * p.num_kv_heads * G;
        const int per_cta = kMergeThreads / 32;
        int mgrid = (items + per_cta - 1) / per_cta;
        if (mgrid > 2 * nruns)
            mgrid = 2 * nruns;
        void* args[] = {&p, &nruns};
        return MmaLauncher<KV, QT, 128, BS, G, 1>::launch_merge_pdl(
            (const void*)paged_decode_merge_kernel<QT, 128, BS, G, 1, kTcUnit>, args, mgrid,
            (size_t)(p.num_seqs + 1) * 4, stream);
    }
};

}  // namespace pkv
