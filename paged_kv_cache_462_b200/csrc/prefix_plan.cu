// Shared-prefix plan of a decode batch (include/pkv_blocks.h, pkv_prefix_plan): which
// sequences read which leading full blocks through one shared table row. Host code only.
#include <algorithm>
#include <cstdint>
#include <unordered_map>
#include <vector>

#include "pkv_blocks.h"

namespace {

struct Batch {
    const int32_t* tables;
    const int32_t* lens;
    int mb;
    int bs;

    // block j of sequence s is full and names a block
    bool full(int s, int j) const
    {
        return j < mb && (long long)(j + 1) * bs <= lens[s] && tables[(size_t)s * mb + j] >= 0;
    }
    int32_t at(int s, int j) const { return tables[(size_t)s * mb + j]; }
};

}  // namespace

extern "C" int pkv_prefix_plan(const int32_t* block_tables, const int32_t* seq_lens, int num_seqs,
                               int max_blocks_per_seq, int block_size, int max_group, int32_t* group_members,
                               int32_t* group_offsets, int32_t* group_tables, int32_t* group_lens,
                               int32_t* shared_blocks, int* num_groups)
try {
    if (!num_groups)
        return PKV_ERR_NULL;
    *num_groups = 0;
    if (num_seqs < 0 || max_blocks_per_seq <= 0 || block_size <= 0 || max_group < 1)
        return PKV_ERR_SHAPE;
    if (!group_offsets)
        return PKV_ERR_NULL;
    group_offsets[0] = 0;
    if (num_seqs == 0)
        return PKV_OK;
    if (!block_tables || !seq_lens || !group_members || !group_tables || !group_lens || !shared_blocks)
        return PKV_ERR_NULL;
    const Batch b{block_tables, seq_lens, max_blocks_per_seq, block_size};

    // buckets by first block, in order of their first sequence
    std::unordered_map<int32_t, int> bucket_of;
    std::vector<std::vector<int>> buckets;
    for (int s = 0; s < num_seqs; ++s) {
        shared_blocks[s] = 0;
        if (!b.full(s, 0))
            continue;
        auto it = bucket_of.find(b.at(s, 0));
        if (it == bucket_of.end()) {
            it = bucket_of.emplace(b.at(s, 0), (int)buckets.size()).first;
            buckets.emplace_back();
        }
        buckets[it->second].push_back(s);
    }

    int ng = 0, nm = 0;
    std::vector<int> active, next;
    for (const std::vector<int>& members : buckets) {
        for (size_t c0 = 0; c0 < members.size(); c0 += (size_t)max_group) {
            const size_t c1 = std::min(members.size(), c0 + (size_t)max_group);
            if (c1 - c0 < 2)
                continue;
            int32_t* row = group_tables + (size_t)ng * max_blocks_per_seq;
            active.assign(members.begin() + c0, members.begin() + c1);
            int j = 0;
            for (; j < max_blocks_per_seq; ++j) {
                // the id most active members hold at j; ties go to the first member's
                int32_t best = -1;
                int best_n = 1;
                for (size_t a = 0; a < active.size(); ++a) {
                    if (!b.full(active[a], j))
                        continue;
                    const int32_t x = b.at(active[a], j);
                    int n = 0;
                    for (int s : active)
                        n += b.full(s, j) && b.at(s, j) == x;
                    if (n > best_n) {
                        best = x;
                        best_n = n;
                    }
                }
                if (best_n < 2)
                    break;
                row[j] = best;
                next.clear();
                for (int s : active)
                    if (b.full(s, j) && b.at(s, j) == best) {
                        next.push_back(s);
                        shared_blocks[s] = j + 1;
                    }
                active.swap(next);
            }
            std::fill(row + j, row + max_blocks_per_seq, -1);
            group_lens[ng] = j * block_size;
            for (size_t i = c0; i < c1; ++i)
                group_members[nm++] = members[i];
            group_offsets[++ng] = nm;
        }
    }
    *num_groups = ng;
    return PKV_OK;
} catch (...) {
    return PKV_BM_HOST_ALLOC;
}

extern "C" int pkv_prefix_pass_inputs(const int32_t* block_tables, const int32_t* seq_lens, int num_seqs,
                                      int max_blocks_per_seq, int block_size, const int32_t* group_members,
                                      const int32_t* group_offsets, int num_groups, const int32_t* shared_blocks,
                                      int query_heads_per_kv_head, int32_t* col_seq, int32_t* col_limit,
                                      int32_t* suffix_tables, int32_t* suffix_lens)
{
    const int Gq = query_heads_per_kv_head;
    if (num_seqs < 0 || num_groups < 0 || max_blocks_per_seq <= 0 || block_size <= 0 || Gq <= 0 || 8 % Gq != 0)
        return PKV_ERR_SHAPE;
    if (num_seqs == 0 && num_groups == 0)
        return PKV_OK;
    if (!block_tables || !seq_lens || !shared_blocks || !suffix_tables || !suffix_lens)
        return PKV_ERR_NULL;
    if (num_groups > 0 && (!group_members || !group_offsets || !col_seq || !col_limit))
        return PKV_ERR_NULL;
    for (int s = 0; s < num_seqs; ++s) {
        const int sh = shared_blocks[s];
        if (sh < 0 || sh > max_blocks_per_seq || (long long)sh * block_size > seq_lens[s])
            return PKV_ERR_SHAPE;
    }
    for (int g = 0; g < num_groups; ++g) {
        const int m0 = group_offsets[g], m1 = group_offsets[g + 1];
        if (m0 < 0 || m1 < m0 || m1 > num_seqs || (m1 - m0) * Gq > 8)
            return PKV_ERR_SHAPE;
        for (int c = 0; c < 8; ++c) {
            const int i = c / Gq;
            const bool used = m0 + i < m1;
            const int s = used ? group_members[m0 + i] : -1;
            if (used && (s < 0 || s >= num_seqs))
                return PKV_ERR_SHAPE;
            col_seq[g * 8 + c] = s;
            col_limit[g * 8 + c] = used ? shared_blocks[s] * block_size : 0;
        }
    }
    for (int s = 0; s < num_seqs; ++s) {
        const int sh = shared_blocks[s];
        const int32_t* row = block_tables + (size_t)s * max_blocks_per_seq;
        int32_t* dst = suffix_tables + (size_t)s * max_blocks_per_seq;
        std::copy(row + sh, row + max_blocks_per_seq, dst);
        std::fill(dst + (max_blocks_per_seq - sh), dst + max_blocks_per_seq, -1);
        suffix_lens[s] = seq_lens[s] - sh * block_size;
    }
    return PKV_OK;
}
