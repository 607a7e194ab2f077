// Host-side block manager of the paged KV cache (include/pkv_blocks.h): FIFO free
// list, per-block reference counts, per-sequence block tables, append with
// allocation and copy on write of a shared last block, and the decode step's
// slot_mapping / block_tables / seq_lens. Host code only (no device calls).
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <deque>
#include <new>
#include <unordered_map>
#include <vector>

#include "pkv_blocks.h"

struct pkv_block_manager {
    int num_blocks;
    int block_size;
    int max_blocks;
    std::deque<int32_t> free_list;   // front = next block handed out
    std::vector<int32_t> refs;       // reference count per block
    struct Seq {
        int len = 0;
        std::vector<int32_t> table;
    };
    std::unordered_map<int64_t, Seq> seqs;

    int32_t take()
    {
        const int32_t b = free_list.front();
        free_list.pop_front();
        refs[b] = 1;
        return b;
    }

    void release(int32_t b)
    {
        if (--refs[b] == 0)
            free_list.push_back(b);
    }

    int append(int64_t id, int64_t* slot, int32_t* cow_src, int32_t* cow_dst)
    {
        *cow_src = *cow_dst = -1;
        auto it = seqs.find(id);
        if (it == seqs.end())
            return PKV_BM_UNKNOWN_SEQ;
        Seq& q = it->second;
        const int off = q.len % block_size;
        if (off == 0) {   // the last block is full (or there is none): a fresh block
            if ((int)q.table.size() >= max_blocks)
                return PKV_BM_TABLE_FULL;
            if (free_list.empty())
                return PKV_BM_NO_BLOCKS;
            q.table.push_back(take());
        } else if (refs[q.table.back()] > 1) {   // shared, partly filled: copy on write
            if (free_list.empty())
                return PKV_BM_NO_BLOCKS;
            const int32_t old = q.table.back();
            const int32_t fresh = take();
            refs[old] -= 1;   // still > 0: another sequence holds it
            q.table.back() = fresh;
            *cow_src = old;
            *cow_dst = fresh;
        }
        *slot = (int64_t)q.table.back() * block_size + off;
        q.len += 1;
        return PKV_OK;
    }

    void write_tables(const int64_t* ids, int n, int32_t* tables, int32_t* lens) const
    {
        for (int i = 0; i < n; ++i) {
            const Seq& q = seqs.at(ids[i]);
            int32_t* row = tables + (size_t)i * max_blocks;
            const size_t used = q.table.size();
            if (used > 0)
                std::memcpy(row, q.table.data(), used * sizeof(int32_t));
            std::fill(row + used, row + max_blocks, -1);
            lens[i] = q.len;
        }
    }
};

extern "C" {

pkv_block_manager* pkv_bm_create(int num_blocks, int block_size, int max_blocks_per_seq)
{
    if (num_blocks <= 0 || block_size <= 0 || max_blocks_per_seq <= 0)
        return nullptr;
    auto* bm = new (std::nothrow) pkv_block_manager;
    if (!bm)
        return nullptr;
    try {
        bm->num_blocks = num_blocks;
        bm->block_size = block_size;
        bm->max_blocks = max_blocks_per_seq;
        bm->refs.assign(num_blocks, 0);
        for (int32_t b = 0; b < num_blocks; ++b)
            bm->free_list.push_back(b);
    } catch (...) {
        delete bm;
        return nullptr;
    }
    return bm;
}

void pkv_bm_destroy(pkv_block_manager* bm) { delete bm; }

int pkv_bm_add(pkv_block_manager* bm, int64_t seq_id, int prompt_len)
try {
    if (!bm)
        return PKV_ERR_NULL;
    if (prompt_len < 0)
        return PKV_ERR_SHAPE;
    if (bm->seqs.count(seq_id))
        return PKV_BM_DUPLICATE_SEQ;
    const long long need = ((long long)prompt_len + bm->block_size - 1) / bm->block_size;
    if (need > bm->max_blocks)
        return PKV_BM_TABLE_FULL;
    if (need > (long long)bm->free_list.size())
        return PKV_BM_NO_BLOCKS;
    pkv_block_manager::Seq q;
    q.len = prompt_len;
    q.table.reserve((size_t)need);
    for (long long i = 0; i < need; ++i)
        q.table.push_back(bm->take());
    bm->seqs.emplace(seq_id, std::move(q));
    return PKV_OK;
} catch (...) {
    return PKV_BM_HOST_ALLOC;
}

int pkv_bm_fork(pkv_block_manager* bm, int64_t parent_id, int64_t child_id)
try {
    if (!bm)
        return PKV_ERR_NULL;
    auto it = bm->seqs.find(parent_id);
    if (it == bm->seqs.end())
        return PKV_BM_UNKNOWN_SEQ;
    if (bm->seqs.count(child_id))
        return PKV_BM_DUPLICATE_SEQ;
    pkv_block_manager::Seq child = it->second;
    for (int32_t b : child.table)
        bm->refs[b] += 1;
    bm->seqs.emplace(child_id, std::move(child));
    return PKV_OK;
} catch (...) {
    return PKV_BM_HOST_ALLOC;
}

int pkv_bm_append(pkv_block_manager* bm, int64_t seq_id, int64_t* slot, int32_t* cow_src, int32_t* cow_dst)
try {
    if (!bm || !slot || !cow_src || !cow_dst)
        return PKV_ERR_NULL;
    return bm->append(seq_id, slot, cow_src, cow_dst);
} catch (...) {
    return PKV_BM_HOST_ALLOC;
}

int pkv_bm_free(pkv_block_manager* bm, int64_t seq_id)
try {
    if (!bm)
        return PKV_ERR_NULL;
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end())
        return PKV_BM_UNKNOWN_SEQ;
    for (int32_t b : it->second.table)
        bm->release(b);
    bm->seqs.erase(it);
    return PKV_OK;
} catch (...) {
    return PKV_BM_HOST_ALLOC;
}

int pkv_bm_num_free(const pkv_block_manager* bm) { return bm ? (int)bm->free_list.size() : -1; }

int pkv_bm_seq_len(const pkv_block_manager* bm, int64_t seq_id)
{
    if (!bm)
        return -1;
    auto it = bm->seqs.find(seq_id);
    return it == bm->seqs.end() ? -1 : it->second.len;
}

int pkv_bm_ref_count(const pkv_block_manager* bm, int block)
{
    if (!bm || block < 0 || block >= bm->num_blocks)
        return -1;
    return bm->refs[block];
}

int pkv_bm_step(pkv_block_manager* bm, const int64_t* seq_ids, int n, int64_t* slot_mapping, int32_t* block_tables,
                int32_t* seq_lens, int32_t* cow_pairs, int* n_cow, int* n_done)
try {
    if (!bm || !n_cow || !n_done)
        return PKV_ERR_NULL;
    *n_cow = 0;
    *n_done = 0;
    if (n < 0)
        return PKV_ERR_SHAPE;
    if (n > 0 && (!seq_ids || !slot_mapping || !block_tables || !seq_lens || !cow_pairs))
        return PKV_ERR_NULL;
    for (int i = 0; i < n; ++i) {
        int32_t src, dst;
        const int st = bm->append(seq_ids[i], slot_mapping + i, &src, &dst);
        if (st != PKV_OK)
            return st;
        if (src >= 0) {
            cow_pairs[2 * *n_cow] = src;
            cow_pairs[2 * *n_cow + 1] = dst;
            *n_cow += 1;
        }
        *n_done = i + 1;
    }
    bm->write_tables(seq_ids, n, block_tables, seq_lens);
    return PKV_OK;
} catch (...) {
    return PKV_BM_HOST_ALLOC;
}

int pkv_bm_tables(const pkv_block_manager* bm, const int64_t* seq_ids, int n, int32_t* block_tables,
                  int32_t* seq_lens)
{
    if (!bm)
        return PKV_ERR_NULL;
    if (n < 0)
        return PKV_ERR_SHAPE;
    if (n > 0 && (!seq_ids || !block_tables || !seq_lens))
        return PKV_ERR_NULL;
    for (int i = 0; i < n; ++i)
        if (!bm->seqs.count(seq_ids[i]))
            return PKV_BM_UNKNOWN_SEQ;
    bm->write_tables(seq_ids, n, block_tables, seq_lens);
    return PKV_OK;
}

}  // extern "C"
