// pkv_validate_tables: host check of a decode batch's tables (include/pkv.h). Host code only.
#include <cstdint>
#include <unordered_set>

#include "pkv_blocks.h"

extern "C" int pkv_validate_tables(const int32_t* block_tables, const int32_t* seq_lens, int num_seqs,
                                   int max_blocks_per_seq, int block_size, int num_blocks,
                                   const int64_t* slot_mapping, int32_t* bad_bits, int32_t* first_bad)
try {
    if (!bad_bits || !first_bad)
        return PKV_ERR_NULL;
    *bad_bits = 0;
    *first_bad = -1;
    if (num_seqs < 0 || max_blocks_per_seq <= 0 || block_size <= 0 || num_blocks <= 0)
        return PKV_ERR_SHAPE;
    if (num_seqs == 0)
        return PKV_OK;
    if (!block_tables || !seq_lens)
        return PKV_ERR_NULL;
    const long long capacity = (long long)max_blocks_per_seq * block_size;
    std::unordered_set<int64_t> used;
    for (int s = 0; s < num_seqs; ++s) {
        int bits = 0;
        long long L = seq_lens[s];
        if (L < 0 || L > capacity) {
            bits |= PKV_DEVERR_SEQ_LEN;
            L = L < 0 ? 0 : capacity;   // the kernels clamp the same way
        }
        const long long nb = (L + block_size - 1) / block_size;
        const int32_t* row = block_tables + (size_t)s * max_blocks_per_seq;
        for (long long j = 0; j < nb; ++j)
            if (row[j] < 0 || row[j] >= num_blocks)
                bits |= PKV_DEVERR_BLOCK_ID;
        if (slot_mapping && slot_mapping[s] >= 0) {
            const int64_t slot = slot_mapping[s];
            if (slot >= (int64_t)num_blocks * block_size || L == 0 ||
                slot / block_size != (int64_t)row[(L - 1) / block_size] || !used.insert(slot).second)
                bits |= PKV_DEVERR_SLOT;
        }
        if (bits && *first_bad < 0)
            *first_bad = s;
        *bad_bits |= bits;
    }
    return PKV_OK;
} catch (...) {
    return PKV_BM_HOST_ALLOC;
}
