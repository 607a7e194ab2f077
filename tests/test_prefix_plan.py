"""Shared-prefix plan of a decode batch: the plain model (oracle/block_model.prefix_plan)
pinned to batches whose sharing is known by construction and to invariants any correct
plan keeps, planted mistakes caught, then the C++ planner (pkv_prefix_plan) checked
against the model on seeded random batches. No GPU."""
import inspect
import textwrap

import numpy as np
import pytest

import workloads as W
from oracle import block_model
from oracle.block_model import OK, BlockModel, prefix_plan


def nblocks(lens, bs):
    return [-(-int(L) // bs) for L in lens]


def constructed(rng, n_groups, size, bs, max_group, share_max=12, loners=3):
    """Groups whose members share the first n_s blocks of one prefix (n_s drawn; 0 = the
    member shares nothing), plus sequences that share with nobody. Tables, lens and the
    groups a correct plan must return: per chunk of max_group sharing members (index
    order), the table is the prefix cut at the second-largest n_s, and each member shares
    min(n_s, that)."""
    tables, lens, expect = [], [], []
    nxt = iter(rng.permutation(100000).tolist())
    for _ in range(n_groups):
        prefix = [next(nxt) for _ in range(share_max)]
        ns = [int(x) for x in rng.integers(0, share_max + 1, size=size)]
        ids = []
        for n in ns:
            L = n * bs + int(rng.integers(1, 3 * bs))      # the shared blocks are full
            own = -(-L // bs) - n
            ids.append(len(tables))
            tables.append(prefix[:n] + [next(nxt) for _ in range(own)])
            lens.append(L)
        sharing = [i for i, n in zip(ids, ns) if n > 0]
        for c0 in range(0, len(sharing), max_group):
            chunk = sharing[c0:c0 + max_group]
            if len(chunk) < 2:
                continue
            depth = sorted(ns[ids.index(s)] for s in chunk)[-2]
            expect.append((chunk, prefix[:depth], [min(ns[ids.index(s)], depth) for s in chunk]))
    for _ in range(loners):
        L = int(rng.integers(1, 5 * bs))
        tables.append([next(nxt) for _ in range(-(-L // bs))])
        lens.append(L)
    mb = max(len(t) for t in tables)
    return [t + [-1] * (mb - len(t)) for t in tables], lens, expect


def check_plan(plan, tables, lens, bs, max_group, refs=None):
    """Invariants: members of a group share its row's blocks, full, in their own tables;
    each row block is held by two or more members; the walk could not go one block deeper;
    a sequence is in one group at most; groups respect max_group; every sequence whose
    full first block another sequence also holds is grouped unless it is a chunk of one."""
    full = lambda s, j: j < len(tables[s]) and (j + 1) * bs <= lens[s] and tables[s][j] >= 0
    seen = set()
    for members, row, shared in plan:
        assert 2 <= len(members) <= max_group and not (seen & set(members))
        seen |= set(members)
        assert len(row) == max(shared)
        for j, b in enumerate(row):
            holders = [s for s, p in zip(members, shared) if p > j]
            assert len(holders) >= 2
            for s in holders:
                assert full(s, j) and tables[s][j] == b
                if refs is not None:
                    assert refs[b] >= 2
        deepest = [s for s, p in zip(members, shared) if p == len(row)]
        ids = [tables[s][len(row)] for s in deepest if full(s, len(row))]
        assert len(ids) == len(set(ids))
        for s, p in zip(members, shared):      # a member stops where its block differs
            if p < len(row):
                assert not full(s, p) or tables[s][p] != row[p]
    first = {}
    for s in range(len(lens)):
        if full(s, 0):
            first.setdefault(tables[s][0], []).append(s)
    for bucket in first.values():
        for i, s in enumerate(bucket):
            lone = i % max_group == 0 and i == len(bucket) - 1
            assert (s in seen) == (len(bucket) > 1 and not lone)


# ------------------------------------------------------------------ model pins

@pytest.mark.parametrize("max_group", [2, 3, 8, 64])
def test_model_recovers_constructed_sharing(max_group):
    rng = np.random.default_rng(max_group)
    for bs in (1, 4, 16):
        tables, lens, expect = constructed(rng, 6, 9, bs, max_group)
        plan = prefix_plan(tables, lens, bs, max_group)
        assert sorted(plan) == sorted(expect)
        check_plan(plan, tables, lens, bs, max_group)


def test_model_counts_full_blocks_only():
    """A 40-token prompt forked three times (block 16): blocks 0 and 1 are full and shared,
    block 2 is shared but holds 8 tokens, so it is read per sequence."""
    m = BlockModel(16, 16, 8)
    assert m.add(0, 40) == OK and all(m.fork(0, c) == OK for c in (1, 2, 3))
    tables = [m.seqs[s][1] for s in range(4)]
    plan = prefix_plan(tables, [40] * 4, 16, 8)
    assert plan == [([0, 1, 2, 3], tables[0][:2], [2, 2, 2, 2])]
    assert prefix_plan(tables, [48] * 4, 16, 8)[0][1] == tables[0]      # 48 tokens: all full


def test_model_ties_and_chunks():
    tables = [[5, 6], [5, 7], [5, 6], [5, 7]]
    assert prefix_plan(tables, [32] * 4, 16, 8) == [([0, 1, 2, 3], [5, 6], [2, 1, 2, 1])]
    five = [[9, 1, 2]] * 5
    assert prefix_plan(five, [48] * 5, 16, 2) == [([0, 1], [9, 1, 2], [3, 3]), ([2, 3], [9, 1, 2], [3, 3])]
    assert prefix_plan(five, [48] * 5, 16, 1) == []
    assert prefix_plan([[1, 2], [3, 4]], [32, 32], 16, 8) == []
    assert prefix_plan([], [], 16, 8) == []
    assert prefix_plan([[4, -1], [4, -1]], [15, 15], 16, 8) == []         # first block not full


def test_model_on_block_manager_batches():
    """Fork trees with appends (copy on write included): every block a plan shares is held
    by two or more tables in the manager's counts."""
    rng = np.random.default_rng(5)
    for trial in range(30):
        bs = int(rng.choice([1, 4, 16]))
        m = BlockModel(400, bs, 64)
        live = []
        for sid in range(int(rng.integers(2, 14))):
            if live and rng.random() < 0.6:
                assert m.fork(live[int(rng.integers(len(live)))], sid) == OK
            else:
                assert m.add(sid, int(rng.integers(0, 6 * bs))) == OK
            live.append(sid)
            for _ in range(int(rng.integers(0, 2 * bs))):
                m.append(live[int(rng.integers(len(live)))])
        tables = [m.seqs[s][1] + [-1] * (64 - len(m.seqs[s][1])) for s in live]
        lens = [m.seqs[s][0] for s in live]
        for mg in (2, 8):
            check_plan(prefix_plan(tables, lens, bs, mg), tables, lens, bs, mg, refs=m.refs)


def test_mixed_prefix_workload_plan():
    """The 256-sequence mixed batch (groups of 8 sharing up to 64 blocks): the plan finds
    the groups the workload built, and reads 33743 blocks instead of 47514."""
    spec = W.config_spec(3)
    lay = W.batch_layout(spec)
    bs, tables, lens = spec.block_size, lay.block_tables.tolist(), lay.seq_lens.tolist()
    plan = prefix_plan(tables, lens, bs, spec.share_group)
    check_plan(plan, tables, lens, bs, spec.share_group)
    want = {}
    for members, _ in lay.groups:
        sharing = [s for s in members if lay.shared_n[s] > 0]
        depth = sorted(int(lay.shared_n[s]) for s in sharing)[-2]
        want[tuple(sharing)] = [min(int(lay.shared_n[s]), depth) for s in sharing]
    assert {tuple(m): p for m, _, p in plan} == want
    shared = np.zeros(len(lens), np.int64)
    for m, _, p in plan:
        shared[m] = p
    nb = np.asarray(nblocks(lens, bs))
    assert (int(nb.sum()), sum(len(r) for _, r, _ in plan) + int((nb - shared).sum())) == (47514, 33743)
    reads = {}
    for mg in (2, 4):
        smaller = prefix_plan(tables, lens, bs, mg)
        check_plan(smaller, tables, lens, bs, mg)
        sh = np.zeros(len(lens), np.int64)
        for m, _, p in smaller:
            sh[m] = p
        reads[mg] = sum(len(r) for _, r, _ in smaller) + int((nb - sh).sum())
    assert reads == {2: 39865, 4: 35791}


# ------------------------------------------------------------------ planted mistakes

MUTANTS = {
    "partial blocks count": ("(j + 1) * bs <= lens[s]", "j * bs < lens[s]"),
    "one holder is enough": ("best, best_n = None, 1", "best, best_n = None, 0"),
    "no chunking": ("chunk = members[c0:c0 + max(1, max_group)]", "chunk = members if c0 == 0 else []"),
    "group-wide depth": ("for s in active:\n                    shared[s] = j + 1",
                         "for s in chunk:\n                    shared[s] = j + 1"),
}


def _mutant(name):
    src = textwrap.dedent(inspect.getsource(block_model.prefix_plan))
    old, new = MUTANTS[name]
    assert src.count(old) == 1, name
    ns = {}
    exec(src.replace(old, new), ns)
    return ns["prefix_plan"]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistakes(name, monkeypatch):
    monkeypatch.setitem(globals(), "prefix_plan", _mutant(name))
    pins = [lambda: test_model_recovers_constructed_sharing(3), test_model_counts_full_blocks_only,
            test_model_ties_and_chunks, test_model_on_block_manager_batches]
    caught = 0
    for pin in pins:
        try:
            pin()
        except (AssertionError, IndexError, KeyError):
            caught += 1
    assert caught >= 1, name


# ------------------------------------------------------------------ C++ planner vs model

@pytest.fixture(scope="module")
def cplan():
    from paged_kv_cache_462_b200 import build
    build.build()
    from paged_kv_cache_462_b200.blocks import prefix_plan as plan
    return plan


@pytest.mark.parametrize("seed", range(8))
def test_cpp_planner_matches_model(cplan, seed):
    rng = np.random.default_rng(900 + seed)
    bs = int(rng.choice([1, 8, 16, 32]))
    n, mb = int(rng.integers(1, 40)), int(rng.integers(1, 12))
    # few distinct ids, so tables collide at every depth; some -1 holes and short lengths
    tables = rng.integers(-1, 5, size=(n, mb)).astype(np.int32)
    tables[:, 0] = rng.integers(0, 3, size=n)
    lens = rng.integers(0, mb * bs + 1, size=n).astype(np.int32)
    for mg in (1, 2, 3, 8, 64):
        want = prefix_plan(tables.tolist(), lens.tolist(), bs, mg)
        got = cplan(tables, lens, bs, mg)
        assert got.groups() == want
        shared = np.zeros(n, np.int64)
        for m, row, p in want:
            shared[m] = p
        assert got.shared.tolist() == shared.tolist()
        assert got.lens.tolist() == [len(row) * bs for _, row, _ in want]


def test_cpp_planner_on_workload_and_guards(cplan):
    lay = W.batch_layout(W.config_spec(3))
    got = cplan(lay.block_tables, lay.seq_lens, 16, 8)
    assert got.groups() == prefix_plan(lay.block_tables.tolist(), lay.seq_lens.tolist(), 16, 8)
    empty = cplan(np.zeros((0, 4), np.int32), np.zeros(0, np.int32), 16, 8)
    assert empty.num_groups == 0
    from paged_kv_cache_462_b200 import PkvError
    with pytest.raises(PkvError):
        cplan(lay.block_tables, lay.seq_lens, 16, 0)
    with pytest.raises(PkvError):
        cplan(lay.block_tables, lay.seq_lens, 0, 8)


# ------------------------------------------------------------------ the two passes' inputs

@pytest.fixture(scope="module")
def pass_inputs():
    from paged_kv_cache_462_b200 import build
    build.build()
    from paged_kv_cache_462_b200.blocks import prefix_pass_inputs
    return prefix_pass_inputs


def test_pass_inputs_layout(cplan, pass_inputs):
    tables = np.array([[5, 6, 7, -1], [5, 6, 9, 3], [5, 8, -1, -1], [2, 3, -1, -1]], np.int32)
    lens = np.array([40, 60, 20, 30], np.int32)
    plan = cplan(tables, lens, 16, 4)                    # Gq = 2: at most 4 members per group
    assert plan.groups() == [([0, 1, 2], [5, 6], [2, 2, 1])]
    col_seq, col_limit, suf_t, suf_l = pass_inputs(tables, lens, 16, plan, 2)
    assert col_seq.tolist() == [[0, 0, 1, 1, 2, 2, -1, -1]]
    assert col_limit.tolist() == [[32, 32, 32, 32, 16, 16, 0, 0]]
    assert suf_t.tolist() == [[7, -1, -1, -1], [9, 3, -1, -1], [8, -1, -1, -1], [2, 3, -1, -1]]
    assert suf_l.tolist() == [8, 28, 4, 30]
    from paged_kv_cache_462_b200 import PkvError
    with pytest.raises(PkvError):                        # 3 members x 4 heads > 8 columns
        pass_inputs(tables, lens, 16, plan, 4)
    with pytest.raises(PkvError):                        # Gq must divide 8
        pass_inputs(tables, lens, 16, plan, 3)


@pytest.mark.parametrize("kv", ["bf16", "e4m3"])
def test_prefix_passes_recombine_to_the_decode(cplan, pass_inputs, kv):
    """Plan a mixed batch with shared prefixes, build both passes' inputs, run each pass through
    the oracle (prefix: the group row, each member limited to its shared tokens; suffix: the
    shifted table), combine by log-sum-exp weights: every row equals the plain decode."""
    import oracle
    b = W.config_batch(3, num_seqs=12, num_heads=8, num_kv_heads=2, head_dim=32, kv_dtype=kv,
                       lengths=("lognormal", 300, 0.6, 20, 900), share_group=4, share_blocks=12,
                       max_blocks_per_seq=60)
    sp, bs = b.spec, b.spec.block_size
    Gq = sp.num_heads // sp.num_kv_heads
    _, kc, vc = oracle.run_step(b)
    dec = lambda q, bt, sl: oracle.paged_decode(q, sp.q_dtype, kc, vc, kv, bt, sl, sp.num_heads, sp.num_kv_heads,
                                                sp.head_dim, bs, b.num_blocks, b.scale, b.k_scale, b.v_scale,
                                                return_lse=True)
    full, full_lse = dec(b.q, b.block_tables, b.seq_lens)
    plan = cplan(b.block_tables, b.seq_lens, bs, 8 // Gq)
    assert plan.num_groups >= 2
    col_seq, col_limit, suf_t, suf_l = pass_inputs(b.block_tables, b.seq_lens, bs, plan, Gq)
    o2, l2 = dec(b.q, suf_t, suf_l)
    o1 = np.zeros_like(o2)
    l1 = np.full(l2.shape, -np.inf)
    for g in range(plan.num_groups):
        for c in range(0, 8, Gq):
            s = int(col_seq[g, c])
            if s < 0:
                continue
            o, l = dec(b.q[s:s + 1], plan.tables[g:g + 1], np.array([col_limit[g, c]], np.int32))
            o1[s], l1[s] = o[0], l[0]
    M = np.maximum(l1, l2)
    w1 = np.where(l1 == -np.inf, 0.0, np.exp(l1 - M))
    w2 = np.where(l2 == -np.inf, 0.0, np.exp(l2 - M))
    comb = (w1[..., None] * o1 + w2[..., None] * o2) / (w1 + w2)[..., None]
    assert np.allclose(comb, full, rtol=0, atol=1e-12)
    assert np.allclose(M + np.log(w1 + w2), full_lse, rtol=0, atol=1e-12)
    saved = sum(len(r) for _, r, _ in plan.groups())
    assert int(plan.shared.sum()) > saved           # the shared blocks are read fewer times


def test_cpp_planner_on_cpp_block_manager(cplan, blocks_cpp):
    """Tables from the C++ block manager (forks, appends with copy on write): every block the
    C++ plan shares has a count of two or more in the C++ manager."""
    rng = np.random.default_rng(44)
    for trial in range(10):
        bs = int(rng.choice([4, 16]))
        c = blocks_cpp.BlockManager(300, bs, 40)
        live = []
        for sid in range(int(rng.integers(3, 12))):
            if live and rng.random() < 0.6:
                assert c.fork(live[int(rng.integers(len(live)))], sid) == 0
            else:
                assert c.add(sid, int(rng.integers(1, 5 * bs))) == 0
            live.append(sid)
            for _ in range(int(rng.integers(0, 2 * bs))):
                c.append(live[int(rng.integers(len(live)))])
        st, tables, lens = c.tables(live)
        assert st == 0
        refs = [c.ref_count(blk) for blk in range(300)]
        for mg in (2, 8):
            plan = cplan(tables, lens, bs, mg)
            check_plan(plan.groups(), tables.tolist(), lens.tolist(), bs, mg, refs=refs)
        c.close()


@pytest.fixture(scope="module")
def blocks_cpp():
    from paged_kv_cache_462_b200 import build
    build.build()
    from paged_kv_cache_462_b200 import blocks
    return blocks
