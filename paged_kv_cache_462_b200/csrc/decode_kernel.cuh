// Paged decode attention for sm_100a.
//
// What it computes: for every sequence s and query head g,
//   out[s][g] = softmax_t(scale * q[s][g] . K_t) V_t  over the seq_lens[s] cached tokens,
// with K_t/V_t of logical token t read from physical block
// block_tables[s][t / block_size], offset t % block_size, of the shared pool
// ("vLLM inference cost optimisation", developer.aliyun.com, sections 2 and 4;
// wzjinhao.cn vLLM write-up, section 2.1: the kernel reads KV block by block
// through the table), and query head g reading KV head g / (num_heads / num_kv_heads)
// (grouped-query attention, Aliyun article, KV-cache sizing with GQA).
//
// How (one launch; no CTA ever waits for another):
//  * Work unit = one (block, kv head) tile: block_size x head_dim elements of K
//    and of V, each one contiguous run of the pool. The tiles of all
//    (sequence, kv head) pairs, sequence-major, are cut into gridDim.x equal
//    runs and CTA c owns run c (one CTA per SM by default). A run may cover
//    several pairs and a pair may span several runs; the part of a pair inside
//    one run is a "segment".
//  * The W warps of a CTA (8, or 4 when 8 stages would not fit) take the run's
//    tiles round-robin (tile k -> warp k % W). Each warp owns P shared-memory stages (K tile + V tile) and is its
//    own producer: lane 0 issues one bulk copy (TMA, non-tensor) per tile half
//    into a stage and re-arms the stage's mbarrier as soon as the warp has
//    finished reading it, so P tiles per warp (up to ~200 KB per SM) are in
//    flight. Block-table entries for the next 32 tiles of the warp are fetched
//    one batch ahead.
//  * Compute stays on the CUDA cores (a decode step is a matrix-vector product
//    per head group: there is no dense contraction to feed tensor cores). A
//    warp covers a tile as TPP tokens x LPT lanes per pass; each lane holds
//    head_dim/LPT elements of the G query rows (pre-scaled by scale*log2(e))
//    and of the G output accumulators in registers, so the whole GQA group
//    shares every K/V byte read. The q.K partial sums of a token are reduced
//    over its LPT lanes by a transposing butterfly that leaves each lane with
//    one head's score; the online softmax keeps its running max until a new
//    block max passes it by 8 (log2 units), so most blocks skip the rescale.
//  * At the end of a segment the W warps merge in shared memory. A segment
//    that covers its whole pair writes the output; otherwise it stores fp32
//    (o, m, l) partials in the workspace and the last run to arrive on the
//    pair's counter (atomic, then reset to zero) merges them with the
//    log-sum-exp rule and writes the output.
//  * Every wait is bounded; a block id outside the pool is skipped and a bad
//    seq_len clamped, both reported in the workspace error word.
#pragma once

#include <cstdint>
#include <type_traits>

#include "device.cuh"
#include "pkv_internal.h"

namespace pkv {

constexpr float kRescaleSlack = 8.0f;  // log2 units
constexpr int kMaxStagesPerWarp = 8;

template <class KV, class QT, int D, int BS, int G>
struct Cfg {
    static constexpr int LPT = G <= 4 ? 8 : 16;                 // lanes per token
    static constexpr int TPP = 32 / LPT;                        // tokens per warp pass
    static constexpr int kElt = KV::kBytes;
    static constexpr int kRowBytes = D * kElt;
    static constexpr int kChunk = (kRowBytes / LPT) >= 16 ? 16 : kRowBytes / LPT;
    static constexpr int kEPC = kChunk / kElt;                  // elements per chunk
    static constexpr int kCPL = kRowBytes / (LPT * kChunk);     // chunks per lane per row
    static constexpr int kEPL = kEPC * kCPL;                    // elements per lane = D / LPT
    static constexpr int kPairs = kEPL / 2;                     // fp32 pairs per lane per row
    static constexpr int kTile = BS * kRowBytes;                // one (block, kv head) tile
    static constexpr int kStageBytes = 2 * kTile;               // K + V
    static constexpr int kIters = BS / TPP;                     // warp passes per tile
    // 8 warps, each with at least one stage, unless the stages do not fit: then 4
    static constexpr int W = (8 * (kStageBytes + 12) + 8 * (G * D + 2 * G) * 4 + 4096 <= kMaxSmemPerBlock) ? 8 : 4;
    static constexpr int kThreads = W * 32;
    static constexpr int kScratchFloats = W * (G * D + 2 * G);
    static_assert(kEPL * LPT == D, "lane split");
    static_assert(kChunk == 4 || kChunk == 8 || kChunk == 16, "chunk size");
    static_assert(kTile % 16 == 0, "bulk copies move multiples of 16 bytes");
    static_assert(BS % TPP == 0, "block size multiple of tokens per pass");
};

// ---- transposing butterfly over the LPT lanes of one token -----------------
// A level with xor distance OFF on an N-entry array: the lower lane of each
// pair keeps entries [0, K), the upper keeps [K, N), K = ceil(N/2); each sends
// the half it drops, so a level costs K shuffles instead of N.
template <int N>
__device__ __forceinline__ void tr_level(const float (&a)[N], float (&r)[(N + 1) / 2], bool upper, int off)
{
    constexpr int K = (N + 1) / 2, F = N - K;
#pragma unroll
    for (int k = 0; k < K; ++k) {
        const float hi = (k < F) ? a[K + k] : 0.f;
        const float send = upper ? a[k] : hi;
        const float keep = upper ? hi : a[k];
        r[k] = keep + __shfl_xor_sync(kFullMask, send, off);
    }
}

template <int N, int OFF>
__device__ __forceinline__ float tr_reduce_from(const float (&a)[N], int j)
{
    float b[(N + 1) / 2];
    tr_level<N>(a, b, (j & OFF) != 0, OFF);
    if constexpr (OFF == 1) {
        static_assert((N + 1) / 2 == 1, "group size at most the lanes per token");
        return b[0];
    } else {
        return tr_reduce_from<(N + 1) / 2, OFF / 2>(b, j);
    }
}

// Head whose full score lane j (0..LPT-1) of a token group holds after the butterfly, or -1.
template <int G, int LPT>
__host__ __device__ constexpr int lane_head(int j)
{
    int lo = 0, hi = G, n = G;
    for (int off = LPT / 2; off >= 1; off >>= 1) {
        const int k = (n + 1) / 2;
        if (j & off)
            lo += k;
        else
            hi = (lo + k < hi) ? lo + k : hi;
        n = k;
    }
    return lo < hi ? lo : -1;
}

template <int G, int LPT>
__host__ __device__ constexpr int head_src_lane(int g)
{
    for (int j = 0; j < LPT; ++j)
        if (lane_head<G, LPT>(j) == g)
            return j;
    return 0;
}

// Byte offset in the cache of global tile x, -2 for a bad block id.
template <int TILE>
__device__ __forceinline__ long long tile_offset(const DecodeParams& p, const int* prefix, int x)
{
    const int s = find_seq(prefix, p.num_seqs, x);
    const int nb = (prefix[s + 1] - prefix[s]) / p.num_kv_heads;
    const int r = x - prefix[s];
    const int h = r / nb, j = r - h * nb;
    const int phys = __ldg(p.block_tables + (long long)s * p.max_blocks_per_seq + j);
    if (phys < 0 || phys >= p.num_blocks) {
        atomicOr(p.err, PKV_DEVERR_BLOCK_ID);
        return -2;
    }
    return ((long long)phys * p.num_kv_heads + h) * TILE;
}

template <class KV, class QT, int D, int BS, int G>
__global__ void __launch_bounds__(Cfg<KV, QT, D, BS, G>::kThreads, 1) paged_decode_kernel(const DecodeParams p)
{
    using C = Cfg<KV, QT, D, BS, G>;
    constexpr int W = C::W;
    constexpr int kThreads = C::kThreads;
    constexpr int LPT = C::LPT;
    const int P = p.stages_per_warp;
    const int S = W * P;

    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);                      // [S]
    int* skip = reinterpret_cast<int*>(full + S);                             // [S]
    volatile int* abort_flag = skip + S;
    volatile int* last_flag = abort_flag + 1;
    int* prefix = const_cast<int*>(last_flag + 1);                            // [num_seqs + 1]
    float* scratch = reinterpret_cast<float*>(
        (reinterpret_cast<uintptr_t>(prefix + p.num_seqs + 1) + 15) & ~uintptr_t(15));
    uint8_t* stages = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(scratch + C::kScratchFloats) + 127) & ~uintptr_t(127));

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int Hkv = p.num_kv_heads;
    const int capacity = p.max_blocks_per_seq * BS;

    // ---- prologue: barriers and the per-sequence tile prefix -----------------
    if (tid == 0) {
        for (int i = 0; i < S; ++i)
            mbar_init(&full[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    bool bad_len = false;
    for (int s = tid; s < p.num_seqs; s += kThreads) {
        int L = p.seq_lens[s];
        if (L < 0 || L > capacity) {
            bad_len = true;
            L = L < 0 ? 0 : capacity;
        }
        prefix[s + 1] = ((L + BS - 1) / BS) * Hkv;
    }
    if (bad_len && blockIdx.x == 0)
        atomicOr(p.err, PKV_DEVERR_SEQ_LEN);
    if (tid == 0)
        prefix[0] = 0;
    __syncthreads();
    if (warp == 0) {
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

    const int total = prefix[p.num_seqs];
    const int nruns = gridDim.x;
    const int per_run = (total + nruns - 1) / nruns;
    const int run_begin = min(total, (int)blockIdx.x * per_run);
    const int run_end = min(total, run_begin + per_run);
    const int ntiles = run_end - run_begin;

    // zero rows of empty sequences (one run per sequence)
    for (int s = blockIdx.x; s < p.num_seqs; s += nruns) {
        if (prefix[s + 1] == prefix[s]) {
            QT* o = reinterpret_cast<QT*>(p.out) + (size_t)s * p.num_heads * D;
            for (int i = tid; i < p.num_heads * D; i += kThreads)
                from_float(0.f, o + i);
        }
    }

    // ---- this warp's copy stream: own tiles k = warp + W*i, stage warp + W*(i % P)
    // lane l holds the cache offset of own tile (batch + l); `ahead` the next batch.
    const int own_count = ntiles > warp ? (ntiles - warp + W - 1) / W : 0;
    long long cur_off = (lane < own_count) ? tile_offset<C::kTile>(p, prefix, run_begin + warp + W * lane) : -1;
    long long ahead_off =
        (32 + lane < own_count) ? tile_offset<C::kTile>(p, prefix, run_begin + warp + W * (32 + lane)) : -1;
    int batch = 0;          // own-tile index held by lane 0 of cur_off
    int next_issue = 0;     // next own-tile index to issue
    bool aborted = false;

    // Issue own tile `next_issue` into its stage; the whole warp calls, lane 0 acts.
    auto issue_next = [&]() {
        const int i = next_issue;
        if (i - batch >= 32) {
            batch += 32;
            cur_off = ahead_off;
            ahead_off = (batch + 32 + lane < own_count)
                            ? tile_offset<C::kTile>(p, prefix, run_begin + warp + W * (batch + 32 + lane))
                            : -1;
        }
        const long long off = __shfl_sync(kFullMask, cur_off, i - batch);
        if (lane == 0) {
            const int st = warp + W * (i % P);
            if (off < 0) {
                skip[st] = 1;
                mbar_arrive(&full[st]);
            } else {
                skip[st] = 0;
                uint8_t* dst = stages + (size_t)st * C::kStageBytes;
                mbar_arrive_expect_tx(&full[st], 2 * C::kTile);
                bulk_copy_g2s(dst, p.k_cache + off, C::kTile, &full[st]);
                bulk_copy_g2s(dst + C::kTile, p.v_cache + off, C::kTile, &full[st]);
            }
        }
        ++next_issue;
    };
    while (next_issue < own_count && next_issue < P)
        issue_next();

    // ---- segments of the run ---------------------------------------------------
    const int tq = lane / LPT;  // token within a warp pass
    const int j = lane % LPT;   // lane within the token's group
    const int myhead = lane_head<G, LPT>(j);
    const int group_base = lane & ~(LPT - 1);
    float* scr_o = scratch;                       // [W][G][D]
    float* scr_m = scratch + W * G * D;           // [W][G]
    float* scr_l = scr_m + W * G;                 // [W][G]
    int own = 0;                                  // own-tile index of this warp's next tile

    int x = run_begin;
    while (x < run_end) {
        const int s = find_seq(prefix, p.num_seqs, x);
        const int nb = (prefix[s + 1] - prefix[s]) / Hkv;
        const int h = (x - prefix[s]) / nb;
        const int pair_begin = prefix[s] + h * nb;
        const int pair_end = pair_begin + nb;
        const int seg_end = min(run_end, pair_end);
        int L = p.seq_lens[s];
        L = L < 0 ? 0 : (L > capacity ? capacity : L);

        // q rows of the group as fp32 pairs, pre-scaled (scale * log2(e) [* k_scale * 2^120])
        float2 q2[G][C::kPairs];
        {
            const QT* qp = reinterpret_cast<const QT*>(p.q) + ((size_t)s * p.num_heads + (size_t)h * G) * D;
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int c = 0; c < C::kCPL; ++c) {
                    float t[C::kEPC];
                    load_q<C::kEPC>(qp + g * D + (c * LPT + j) * C::kEPC, t);
#pragma unroll
                    for (int i = 0; i < C::kEPC / 2; ++i)
                        q2[g][c * (C::kEPC / 2) + i] = make_float2(t[2 * i] * p.q_scale, t[2 * i + 1] * p.q_scale);
                }
        }
        float2 o2[G][C::kPairs];
        float m[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            m[g] = -INFINITY;
#pragma unroll
            for (int e = 0; e < C::kPairs; ++e)
                o2[g][e] = make_float2(0.f, 0.f);
        }
        float l_own = 0.f, m_own = -INFINITY;

        // own tiles inside [x, seg_end): tile k = warp + W*own; two tiles per step
        // give each warp two independent q.K / p.V streams and one shared max reduction
        auto wait_tile = [&](int o) {
            const int st = warp + W * (o % P);
            const uint32_t parity = (o / P) & 1;
            bool ok = true;
            if (!aborted)
                ok = !*abort_flag && mbar_wait_bounded(&full[st], parity);
            if (__any_sync(kFullMask, !ok)) {   // one decision for the whole warp
                if (!aborted && lane == 0 && !*abort_flag) {
                    *abort_flag = 1;
                    atomicOr(p.err, PKV_DEVERR_TIMEOUT);
                }
                aborted = true;
            }
        };
        auto tiles = [&](auto nt_tag) {
            constexpr int NT = decltype(nt_tag)::value;
            const uint8_t* kt[NT];
            int valid[NT];
            bool live[NT];
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const int st = warp + W * ((own + t) % P);
                const int jb = run_begin + warp + W * (own + t) - pair_begin;   // logical block
                valid[t] = min(BS, L - jb * BS);
                live[t] = !aborted && skip[st] == 0 && valid[t] > 0;        // warp-uniform
                kt[t] = stages + (size_t)st * C::kStageBytes;
            }
            // ---- scores for this lane's head and tokens tq + TPP*it of each tile
            float sc[NT][C::kIters];
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int it = 0; it < C::kIters; ++it) {
                    const uint8_t* row = kt[t] + (tq + C::TPP * it) * C::kRowBytes;
                    float2 acc2[G];
#pragma unroll
                    for (int g = 0; g < G; ++g)
                        acc2[g] = make_float2(0.f, 0.f);
#pragma unroll
                    for (int c = 0; c < C::kCPL; ++c) {
                        float2 kf[C::kEPC / 2];
                        load_widen2<KV, C::kChunk>(row + (c * LPT + j) * C::kChunk, kf);
#pragma unroll
                        for (int i = 0; i < C::kEPC / 2; ++i)
#pragma unroll
                            for (int g = 0; g < G; ++g)
                                acc2[g] = __ffma2_rn(q2[g][c * (C::kEPC / 2) + i], kf[i], acc2[g]);
                    }
                    float acc[G];
#pragma unroll
                    for (int g = 0; g < G; ++g)
                        acc[g] = acc2[g].x + acc2[g].y;
                    const float v = tr_reduce_from<G, LPT / 2>(acc, j);
                    sc[t][it] = (live[t] && tq + C::TPP * it < valid[t]) ? v : -INFINITY;
                }
            // ---- running max per head (lazy: move it only when the block max passes it by the slack)
            float bm = sc[0][0];
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int it = 0; it < C::kIters; ++it)
                    bm = fmaxf(bm, sc[t][it]);
#pragma unroll
            for (int off = LPT; off < 32; off <<= 1)
                bm = fmaxf(bm, __shfl_xor_sync(kFullMask, bm, off));
            bool moved = false;
            float alpha[G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float b = __shfl_sync(kFullMask, bm, head_src_lane<G, LPT>(g));
                const bool up = b > m[g] + kRescaleSlack;
                const float mn = up ? b : m[g];
                alpha[g] = up ? fast_exp2(m[g] - mn) : 1.f;
                moved |= up;
                m[g] = mn;
            }
            if (moved) {
#pragma unroll
                for (int g = 0; g < G; ++g) {
#pragma unroll
                    for (int e = 0; e < C::kPairs; ++e)
                        o2[g][e] = make_float2(o2[g][e].x * alpha[g], o2[g][e].y * alpha[g]);
                    if (g == myhead) {
                        l_own *= alpha[g];
                        m_own = m[g];
                    }
                }
            }
            float pr[NT][C::kIters];
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int it = 0; it < C::kIters; ++it) {
                    pr[t][it] = (sc[t][it] == -INFINITY) ? 0.f : fast_exp2(sc[t][it] - m_own);
                    l_own += pr[t][it];
                }
            // ---- o += p V for every head of the group
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                if (!live[t])
                    continue;
                const uint8_t* vt = kt[t] + C::kTile;
#pragma unroll
                for (int it = 0; it < C::kIters; ++it) {
                    float2 pg[G];
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const float pv = __shfl_sync(kFullMask, pr[t][it], group_base | head_src_lane<G, LPT>(g));
                        pg[g] = make_float2(pv, pv);
                    }
                    if (tq + C::TPP * it < valid[t]) {
                        const uint8_t* row = vt + (tq + C::TPP * it) * C::kRowBytes;
#pragma unroll
                        for (int c = 0; c < C::kCPL; ++c) {
                            float2 vf[C::kEPC / 2];
                            load_widen2<KV, C::kChunk>(row + (c * LPT + j) * C::kChunk, vf);
#pragma unroll
                            for (int i = 0; i < C::kEPC / 2; ++i)
#pragma unroll
                                for (int g = 0; g < G; ++g)
                                    o2[g][c * (C::kEPC / 2) + i] =
                                        __ffma2_rn(pg[g], vf[i], o2[g][c * (C::kEPC / 2) + i]);
                        }
                    }
                }
            }
        };
        while (own < own_count && run_begin + warp + W * own < seg_end) {
            const bool two = own + 1 < next_issue && run_begin + warp + W * (own + 1) < seg_end;
            wait_tile(own);
            if (two) {
                wait_tile(own + 1);
                tiles(std::integral_constant<int, 2>{});
            } else {
                tiles(std::integral_constant<int, 1>{});
            }
            // the consumed stages are free again: refill them with this warp's tiles own + P (+1)
            __syncwarp();
            const int done = two ? 2 : 1;
            for (int r = 0; r < done; ++r) {
                if (!aborted && next_issue < own_count) {
                    fence_proxy_async_smem();
                    issue_next();
                }
            }
            own += done;
        }

        // ---- fold the token groups of the warp, then merge the warps
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < C::kPairs; ++e) {
                float2 v = o2[g][e];
#pragma unroll
                for (int off = LPT; off < 32; off <<= 1) {
                    v.x += __shfl_xor_sync(kFullMask, v.x, off);
                    v.y += __shfl_xor_sync(kFullMask, v.y, off);
                }
                o2[g][e] = v;
            }
#pragma unroll
        for (int off = LPT; off < 32; off <<= 1)
            l_own += __shfl_xor_sync(kFullMask, l_own, off);
        if (tq == 0) {
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int e = 0; e < C::kPairs; ++e) {
                    const int d = ((2 * e / C::kEPC) * LPT + j) * C::kEPC + (2 * e % C::kEPC);
                    *reinterpret_cast<float2*>(&scr_o[(warp * G + g) * D + d]) = o2[g][e];
                }
            if (myhead >= 0)
                scr_l[warp * G + myhead] = l_own;
        }
        if (lane == 0)
#pragma unroll
            for (int g = 0; g < G; ++g)
                scr_m[warp * G + g] = m[g];
        __syncthreads();

        const int pair = s * Hkv + h;
        const int first_run = pair_begin / per_run;
        const int last_run = (pair_end - 1) / per_run;
        const bool whole = (first_run == last_run);
        QT* out = reinterpret_cast<QT*>(p.out) + ((size_t)s * p.num_heads + (size_t)h * G) * D;
        float* part = p.partials + (size_t)(blockIdx.x + pair) * p.slot_floats;

        for (int idx = tid; idx < G * D; idx += kThreads) {
            const int g = idx / D, d = idx - g * D;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < W; ++w)
                M = fmaxf(M, scr_m[w * G + g]);
            float os = 0.f, ls = 0.f;
            if (M != -INFINITY) {
#pragma unroll
                for (int w = 0; w < W; ++w) {
                    const float mw = scr_m[w * G + g];
                    const float a = (mw == -INFINITY) ? 0.f : fast_exp2(mw - M);
                    os = fmaf(a, scr_o[(w * G + g) * D + d], os);
                    ls = fmaf(a, scr_l[w * G + g], ls);
                }
            }
            if (whole) {
                from_float(ls > 0.f ? (os * p.v_scale) / ls : 0.f, out + g * D + d);
            } else {
                part[g * D + d] = os;
                if (d == 0) {
                    part[G * D + g] = M;
                    part[G * D + G + g] = ls;
                }
            }
        }

        if (!whole) {
            __threadfence();
            __syncthreads();
            if (tid == 0) {
                const int arrived = atomicAdd(&p.counters[pair], 1);
                const int last = (arrived == last_run - first_run) ? 1 : 0;
                if (last)
                    p.counters[pair] = 0;
                *last_flag = last;
            }
            __syncthreads();
            if (*last_flag) {
                __threadfence();
                for (int idx = tid; idx < G * D; idx += kThreads) {
                    const int g = idx / D, d = idx - g * D;
                    float M = -INFINITY;
                    for (int c = first_run; c <= last_run; ++c)
                        M = fmaxf(M, __ldcg(p.partials + (size_t)(c + pair) * p.slot_floats + G * D + g));
                    float os = 0.f, ls = 0.f;
                    if (M != -INFINITY) {
                        for (int c = first_run; c <= last_run; ++c) {
                            const float* q = p.partials + (size_t)(c + pair) * p.slot_floats;
                            const float mc = __ldcg(q + G * D + g);
                            const float a = (mc == -INFINITY) ? 0.f : fast_exp2(mc - M);
                            os = fmaf(a, __ldcg(q + g * D + d), os);
                            ls = fmaf(a, __ldcg(q + G * D + G + g), ls);
                        }
                    }
                    from_float(ls > 0.f ? (os * p.v_scale) / ls : 0.f, out + g * D + d);
                }
            }
        }
        __syncthreads();  // scratch and the flag are reused by the next segment
        x = seg_end;
    }

    // An aborted warp lets its copies still in flight land before the CTA exits.
    if (aborted && lane == 0) {
        for (int i = max(0, next_issue - P); i < next_issue; ++i) {
            const int st = warp + W * (i % P);
            if (!skip[st])
                (void)mbar_wait_bounded(&full[st], (i / P) & 1);
        }
    }
}

// ---------------------------------------------------------------- host side

template <class KV, class QT, int D, int BS, int G>
struct DecodeLauncher {
    using C = Cfg<KV, QT, D, BS, G>;

    static size_t fixed_smem(int num_seqs)
    {
        size_t b = 16;                                             // two flags (+ slack)
        b += (size_t)(num_seqs + 1) * 4 + 16;                      // prefix (+ alignment)
        b += (size_t)C::kScratchFloats * 4 + 128;                  // merge scratch (+ alignment)
        return b;
    }

    static int stages_per_warp(int num_seqs)
    {
        const long long room = (long long)kMaxSmemPerBlock - (long long)fixed_smem(num_seqs);
        const long long per = (long long)C::W * (C::kStageBytes + 12);   // stage + barrier + skip flag
        long long P = room / per;
        if (P > kMaxStagesPerWarp)
            P = kMaxStagesPerWarp;
        return (int)P;
    }

    static size_t smem_bytes(int num_seqs, int P)
    {
        return fixed_smem(num_seqs) + (size_t)C::W * P * (C::kStageBytes + 12);
    }

    static int occupancy(int num_seqs)
    {
        const int P = stages_per_warp(num_seqs);
        if (P < 1)
            return 0;
        int n = 0;
        auto kern = paged_decode_kernel<KV, QT, D, BS, G>;
        const size_t smem = smem_bytes(num_seqs, P);
        if (!ensure_smem_attribute((const void*)kern, smem))
            return 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, C::kThreads, smem) != cudaSuccess)
            return 0;
        return n;
    }

    static int launch(DecodeParams p, int nruns, cudaStream_t stream)
    {
        auto kern = paged_decode_kernel<KV, QT, D, BS, G>;
        const int P = stages_per_warp(p.num_seqs);
        if (P < 1)
            return PKV_ERR_SHAPE;
        const size_t smem = smem_bytes(p.num_seqs, P);
        if (!ensure_smem_attribute((const void*)kern, smem))
            return PKV_ERR_LAUNCH;
        p.stages_per_warp = P;
        // E4M3 codes are widened to fp32 with a 2^-120 bias (see device.cuh): fold 2^120 into the scales
        p.q_scale = p.scale * kLog2e * (KV::kBytes == 1 ? p.k_scale * KV::kUnbias : 1.0f);
        p.v_scale = KV::kBytes == 1 ? p.v_scale_in * KV::kUnbias : 1.0f;
        kern<<<nruns, C::kThreads, smem, stream>>>(p);
        return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_LAUNCH;
    }
};

template <class KV, class QT, int D, int BS>
inline int dispatch_group(int G, const DecodeParams& p, int nruns, cudaStream_t st, int* occ)
{
    switch (G) {
#define PKV_G(GV)                                                            \
    case GV:                                                                 \
        if (occ) {                                                           \
            *occ = DecodeLauncher<KV, QT, D, BS, GV>::occupancy(p.num_seqs); \
            return PKV_OK;                                                   \
        }                                                                    \
        return DecodeLauncher<KV, QT, D, BS, GV>::launch(p, nruns, st);
        PKV_G(1)
        PKV_G(2)
        PKV_G(4)
        PKV_G(5)
        PKV_G(8)
#undef PKV_G
    default:
        return PKV_ERR_SHAPE;
    }
}

template <class KV, class QT, int D>
inline int dispatch_bs(int BS, int G, const DecodeParams& p, int nruns, cudaStream_t st, int* occ)
{
    switch (BS) {
    case 8:
        return dispatch_group<KV, QT, D, 8>(G, p, nruns, st, occ);
    case 16:
        return dispatch_group<KV, QT, D, 16>(G, p, nruns, st, occ);
    case 32:
        return dispatch_group<KV, QT, D, 32>(G, p, nruns, st, occ);
    default:
        return PKV_ERR_SHAPE;
    }
}

template <class KV, class QT>
inline int dispatch_d(int D, int BS, int G, const DecodeParams& p, int nruns, cudaStream_t st, int* occ)
{
    switch (D) {
    case 64:
        return dispatch_bs<KV, QT, 64>(BS, G, p, nruns, st, occ);
    case 128:
        return dispatch_bs<KV, QT, 128>(BS, G, p, nruns, st, occ);
    default:
        return PKV_ERR_SHAPE;
    }
}

}  // namespace pkv
