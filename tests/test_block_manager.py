"""Host block manager: the plain model pinned to the pages' example and to invariants that
any correct pool must keep, then the C++ manager (include/pkv_blocks.h) checked against
the model on seeded random operation sequences. No GPU."""
import os

import numpy as np
import pytest

from oracle.block_model import NO_BLOCKS, OK, TABLE_FULL, UNKNOWN_SEQ, DUPLICATE_SEQ, BlockModel

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "aliyun_s4_block_table.txt")


def golden_table():
    rows = [l.split() for l in open(GOLDEN) if l.strip() and not l.startswith("#")]
    return [int(p) for _, p in sorted((int(a), int(b)) for a, b in rows)]


def check_invariants(m: BlockModel):
    """Counts equal table occurrences; the free list is exactly the unreferenced blocks;
    each table holds ceil(len / bs) blocks."""
    occ = [0] * m.num_blocks
    for length, table in m.seqs.values():
        assert len(table) == -(-length // m.bs)
        for b in table:
            occ[b] += 1
    assert occ == m.refs
    free = list(m.free)
    assert len(set(free)) == len(free)
    assert sorted(free) == [b for b in range(m.num_blocks) if m.refs[b] == 0]


# ------------------------------------------------------------------ model pins

def test_model_reproduces_the_pages_block_table():
    """Pool of 20 blocks of 16 tokens; 20 one-block requests, then requests 7, 2, 19, 4 finish:
    a 60-token request gets the worked example's table 0->7, 1->2, 2->19, 3->4."""
    m = BlockModel(20, 16, 8)
    for i in range(20):
        assert m.add(i, 16) == OK
    for i in (7, 2, 19, 4):
        assert m.free_seq(i) == OK
    assert m.add(100, 60) == OK
    assert m.seqs[100][1] == golden_table()
    st, slot, src, dst = m.append(100)           # position 60: logical block 3, offset 12
    assert (st, slot, src, dst) == (OK, 4 * 16 + 12, -1, -1)
    check_invariants(m)


def test_model_fork_shares_and_copy_on_write_splits():
    m = BlockModel(8, 4, 8)
    assert m.add(1, 6) == OK                      # blocks 0, 1; block 1 holds 2 of 4 tokens
    assert m.fork(1, 2) == OK
    assert m.refs[:2] == [2, 2]
    st, slot, src, dst = m.append(2)              # the child writes into the shared, partly filled block
    assert (st, src, dst) == (OK, 1, 2) and slot == 2 * 4 + 2
    assert m.seqs[1][1] == [0, 1] and m.seqs[2][1] == [0, 2]
    assert m.refs[:3] == [2, 1, 1]
    st, slot, src, dst = m.append(1)              # the parent is now the only holder: no copy
    assert (st, slot, src, dst) == (OK, 1 * 4 + 2, -1, -1)
    check_invariants(m)


def test_model_full_last_block_needs_no_copy():
    m = BlockModel(8, 4, 8)
    assert m.add(1, 8) == OK and m.fork(1, 2) == OK
    st, slot, src, dst = m.append(2)
    assert (st, src, dst) == (OK, -1, -1) and slot == 2 * 4 + 0
    assert m.refs[:3] == [2, 2, 1]
    check_invariants(m)


def test_model_errors_change_nothing():
    m = BlockModel(2, 4, 2)
    assert m.add(1, 9) == TABLE_FULL and m.add(1, 8) == OK
    assert m.append(1)[0] == TABLE_FULL
    assert m.add(2, 1) == NO_BLOCKS
    assert m.add(1, 1) == DUPLICATE_SEQ and m.fork(5, 6) == UNKNOWN_SEQ and m.append(7)[0] == UNKNOWN_SEQ
    assert m.seqs[1] == [8, [0, 1]] and list(m.free) == []
    m2 = BlockModel(3, 4, 4)
    assert m2.add(1, 3) == OK and m2.fork(1, 2) == OK and m2.add(3, 8) == OK
    assert m2.append(2)[0] == NO_BLOCKS            # copy on write needs a block: none free
    assert m2.seqs[2] == [3, [0]] and m2.refs == [2, 1, 1]


def _random_ops(m, rng, n_ops, ids):
    """Random add/fork/append/step/free; yields after every op (for the invariant checks)."""
    live = []
    for _ in range(n_ops):
        r = rng.random()
        if r < 0.2 or not live:
            sid = next(ids)
            if m.add(sid, int(rng.integers(0, 40))) == OK:
                live.append(sid)
        elif r < 0.35:
            sid = next(ids)
            if m.fork(live[int(rng.integers(len(live)))], sid) == OK:
                live.append(sid)
        elif r < 0.7:
            m.append(live[int(rng.integers(len(live)))])
        elif r < 0.85:
            m.step(list(rng.permutation(live))[: int(rng.integers(1, len(live) + 1))])
        else:
            m.free_seq(live.pop(int(rng.integers(len(live)))))
        yield


def test_model_invariants_and_unique_step_slots():
    """Every step's slots are distinct, and each lies in a block that only its own sequence
    holds (so writing the new token cannot show through another sequence's table)."""
    rng = np.random.default_rng(7)
    for trial in range(20):
        m = BlockModel(int(rng.integers(4, 40)), int(rng.choice([1, 4, 16])), 8)
        ids = iter(range(10 ** 6))
        for _ in _random_ops(m, rng, 300, ids):
            check_invariants(m)
        live = list(m.seqs)
        if live:
            st, slots, tables, lens, cows, n_done = m.step(live)
            done = slots[:n_done]
            assert len(set(done)) == len(done)
            for s in done:
                assert m.refs[s // m.bs] == 1
            check_invariants(m)


class _NoCow(BlockModel):
    def append(self, sid):
        if sid not in self.seqs:
            return UNKNOWN_SEQ, -1, -1, -1
        length, table = self.seqs[sid]
        if length % self.bs == 0:
            if not self.free:
                return NO_BLOCKS, -1, -1, -1
            table.append(self._take())
        self.seqs[sid][0] = length + 1
        return OK, table[-1] * self.bs + length % self.bs, -1, -1


class _LifoFree(BlockModel):
    def _take(self):
        b = self.free.pop()
        self.refs[b] = 1
        return b


class _LeakOnFree(BlockModel):
    def free_seq(self, sid):
        if sid not in self.seqs:
            return UNKNOWN_SEQ
        for b in self.seqs.pop(sid)[1]:
            self.refs[b] -= 1
        return OK


@pytest.mark.parametrize("mutant", [_NoCow, _LifoFree, _LeakOnFree])
def test_pins_catch_planted_mistakes(mutant):
    """Each plausible mistake fails at least one of the checks above."""
    def fails(fn):
        try:
            fn()
        except (AssertionError, KeyError, IndexError):
            return True
        return False

    def worked_example():
        m = mutant(20, 16, 8)
        for i in range(20):
            m.add(i, 16)
        for i in (7, 2, 19, 4):
            m.free_seq(i)
        m.add(100, 60)
        assert m.seqs[100][1] == golden_table()
        check_invariants(m)

    def unique_slots():
        rng = np.random.default_rng(3)
        for _ in range(10):
            m = mutant(int(rng.integers(4, 40)), int(rng.choice([1, 4, 16])), 8)
            ids = iter(range(10 ** 6))
            for _ in _random_ops(m, rng, 200, ids):
                check_invariants(m)
            st, slots, *_rest, n_done = m.step(list(m.seqs))
            assert len(set(slots[:n_done])) == n_done
            for s in slots[:n_done]:
                assert m.refs[s // m.bs] == 1

    assert fails(worked_example) or fails(unique_slots)


# ------------------------------------------------------------------ C++ manager vs model

@pytest.fixture(scope="module")
def blocks_mod():
    from paged_kv_cache_462_b200 import build
    build.build()
    from paged_kv_cache_462_b200 import blocks
    return blocks


@pytest.mark.parametrize("seed", range(6))
def test_cpp_manager_matches_model(blocks_mod, seed):
    rng = np.random.default_rng(100 + seed)
    nb, bs, mb = int(rng.integers(3, 64)), int(rng.choice([1, 8, 16, 32])), int(rng.integers(2, 12))
    m = BlockModel(nb, bs, mb)
    c = blocks_mod.BlockManager(nb, bs, mb)
    live, next_id = [], 0
    for _ in range(600):
        r = rng.random()
        if r < 0.2 or not live:
            L = int(rng.integers(0, bs * mb + 2))
            assert c.add(next_id, L) == m.add(next_id, L)
            if next_id in m.seqs:
                live.append(next_id)
            next_id += 1
        elif r < 0.35:
            p = live[int(rng.integers(len(live)))]
            assert c.fork(p, next_id) == m.fork(p, next_id)
            live.append(next_id)
            next_id += 1
        elif r < 0.65:
            s = live[int(rng.integers(len(live)))]
            assert c.append(s) == m.append(s)
        elif r < 0.85:
            ids = [int(x) for x in rng.permutation(live)[: int(rng.integers(1, len(live) + 1))]]
            st, slots, tables, lens, cows, n_done = c.step(ids)
            mst, mslots, mtables, mlens, mcows, mdone = m.step(ids)
            assert (st, n_done) == (mst, mdone)
            assert slots[:n_done].tolist() == mslots[:n_done]
            assert [tuple(p) for p in cows.tolist()] == mcows
            if st == 0:
                assert tables.tolist() == mtables and lens.tolist() == mlens
        else:
            s = live.pop(int(rng.integers(len(live))))
            assert c.free(s) == m.free_seq(s)
        assert c.num_free() == len(m.free)
        for b in range(nb):
            assert c.ref_count(b) == m.refs[b]
    st, tables, lens = c.tables(live)
    assert st == 0
    for i, s in enumerate(live):
        assert lens[i] == m.seqs[s][0] and tables[i].tolist()[: len(m.seqs[s][1])] == m.seqs[s][1]
    assert c.append(10 ** 9)[0] == UNKNOWN_SEQ and c.free(10 ** 9) == UNKNOWN_SEQ
    c.close()
