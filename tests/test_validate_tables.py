"""pkv_validate_tables: the host check of a batch's tables (no GPU). Each case plants one known
problem in a clean batch and expects exactly its bit and the first sequence it affects."""
import numpy as np
import pytest

import paged_kv_cache_462_b200 as pkv
import workloads as W

BLOCK_ID, SEQ_LEN, SLOT = pkv.DEVERR_BLOCK_ID, pkv.DEVERR_SEQ_LEN, pkv.DEVERR_SLOT


@pytest.fixture(scope="module")
def batch():
    from paged_kv_cache_462_b200 import build
    build.build()
    return W.config_batch(3, num_seqs=24)


def _check(b, tables=None, lens=None, slots=None):
    return pkv.validate_tables(b.block_tables if tables is None else tables,
                               b.seq_lens if lens is None else lens, b.spec.block_size, b.num_blocks,
                               b.new_slots if slots is None else slots)


def test_generated_batches_are_clean(batch):
    assert _check(batch) == (0, -1)
    for cfg in (0, 1, 2, 4):
        b = W.config_batch(cfg) if cfg != 2 else W.config_batch(2, num_seqs=4)
        assert pkv.validate_tables(b.block_tables, b.seq_lens, b.spec.block_size, b.num_blocks, b.new_slots) == (0, -1)


def test_block_id_outside_the_pool(batch):
    t = batch.block_tables.copy()
    t[5, 0] = batch.num_blocks                       # one past the pool
    assert _check(batch, tables=t) == (BLOCK_ID, 5)
    t = batch.block_tables.copy()
    t[7, 1] = -3
    assert _check(batch, tables=t) == (BLOCK_ID, 7)


def test_entries_past_the_length_are_not_read(batch):
    t = batch.block_tables.copy()
    nb = -(-int(batch.seq_lens[2]) // batch.spec.block_size)
    t[2, nb:] = 10 ** 9                              # padding past ceil(L / bs): never read
    assert _check(batch, tables=t) == (0, -1)


def test_seq_len_outside_the_table(batch):
    sl = batch.seq_lens.copy()
    sl[9] = batch.max_blocks_per_seq * batch.spec.block_size + 1
    bits, first = _check(batch, lens=sl, slots=np.full_like(batch.new_slots, -1))
    # the kernels clamp the length to the table: the -1 padding then counts as bad entries too
    assert bits == SEQ_LEN | BLOCK_ID and first == 9
    sl = batch.seq_lens.copy()
    sl[11] = -1                                      # clamped to 0: nothing read
    assert _check(batch, lens=sl, slots=np.full_like(batch.new_slots, -1)) == (SEQ_LEN, 11)


def test_slot_rules(batch):
    bs = batch.spec.block_size
    s = batch.new_slots.copy()
    s[3] = batch.num_blocks * bs                     # past the pool
    assert _check(batch, slots=s) == (SLOT, 3)
    s = batch.new_slots.copy()
    s[4] = int(batch.block_tables[4, 0]) * bs        # a block that is not the one holding position L-1
    assert int(batch.seq_lens[4]) > bs
    assert _check(batch, slots=s) == (SLOT, 4)
    s = batch.new_slots.copy()
    s[6] = s[1]                                      # two sequences, one slot
    assert _check(batch, slots=s)[0] == SLOT
    s = batch.new_slots.copy()
    s[8] = -1                                        # a negative slot appends nothing: fine
    assert _check(batch, slots=s) == (0, -1)


def test_several_problems_report_every_bit_and_the_first_sequence(batch):
    t = batch.block_tables.copy()
    t[12, 0] = -1
    sl = batch.seq_lens.copy()
    sl[10] = 10 ** 6
    bits, first = _check(batch, tables=t, lens=sl, slots=np.full_like(batch.new_slots, -1))
    assert bits == BLOCK_ID | SEQ_LEN and first == 10
