"""Shared-prefix decode (prefix pass over each group's shared blocks, suffix pass over each
sequence's own blocks, log-sum-exp merge) against the CPU oracle's plain decode, through the C ABI.

Prefix caching reuses whole blocks, so sequences holding the same physical block hold the same
tokens there (wzjinhao.cn vLLM write-up, section 2.3; "vLLM inference cost optimisation",
section 11): attention over the shared blocks read once per group must equal each sequence's
ordinary attention over its own table. Tolerances as for the plain decode (1e-2 bf16, 3e-2 8-bit).
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_462_b200 as pkv
import workloads as W
from gpu_harness import TOL, GpuStep, cache_bytes, max_err
from paged_kv_cache_462_b200 import blocks

pytestmark = pytest.mark.gpu


def _plan(b, max_group):
    plan = blocks.prefix_plan(b.block_tables, b.seq_lens, b.spec.block_size, max_group)
    return plan, pkv.DevicePrefixPlan(plan, max_group)


def _shared_decode(g, dplan, parts=0, step=False):
    b = g.b
    sp = b.spec
    ws = pkv.new_shared_prefix_workspace(b.num_seqs, sp.num_heads, sp.num_kv_heads, sp.head_dim, dplan.num_groups,
                                         parts)
    out = torch.full_like(g.q, float("nan"))
    if step:
        pkv.paged_decode_step_shared_prefix(out, g.q, g.kc, g.vc, g.bt, g.sl, dplan, g.new_k, g.new_v, g.new_slots,
                                            float(b.scale), float(b.k_scale), float(b.v_scale), parts, ws)
    else:
        pkv.paged_attention_decode_shared_prefix(out, g.q, g.kc, g.vc, g.bt, g.sl, dplan, float(b.scale),
                                                 float(b.k_scale), float(b.v_scale), parts, ws)
    torch.cuda.synchronize()
    return out, pkv.read_device_error(ws)


@pytest.mark.parametrize("kv", ["bf16", "e4m3", "e5m2", "int8"])
@pytest.mark.parametrize("parts", [0, 7, 64])
def test_mixed_prefix_batch_every_output(kv, parts):
    """Config 3's distributions cut down to 24 sequences (3 groups of 8 sharing up to 64 blocks)."""
    b = W.config_batch(3, num_seqs=24, kv_dtype=kv)
    ref, okc, ovc = oracle.run_step(b)
    g = GpuStep(b)
    g.append()
    plan, dplan = _plan(b, 8)
    assert plan.num_groups >= 3 and int(plan.shared.max()) > 0
    out, err = _shared_decode(g, dplan, parts)
    assert err == 0
    assert max_err(out, ref) <= TOL[kv]


@pytest.mark.parametrize("kv", ["bf16", "e4m3"])
def test_fused_step_with_shared_prefix(kv):
    """The append rides in the suffix pass: caches equal the oracle's byte for byte."""
    b = W.config_batch(3, num_seqs=16, kv_dtype=kv)
    ref, okc, ovc = oracle.run_step(b)
    g = GpuStep(b)                                   # history only; the step appends
    _, dplan = _plan(b, 8)
    out, err = _shared_decode(g, dplan, 0, step=True)
    assert err == 0
    assert np.array_equal(cache_bytes(g.kc), okc) and np.array_equal(cache_bytes(g.vc), ovc)
    assert max_err(out, ref) <= TOL[kv]


def test_no_groups_is_the_plain_decode_bit_for_bit():
    """A plan without groups (max_group 1) runs the plain decode's kernel and merge: same bits."""
    b = W.config_batch(3, num_seqs=16)
    g = GpuStep(b)
    g.append()
    ref = g.decode(7).clone()
    plan, dplan = _plan(b, 1)
    assert plan.num_groups == 0
    out, err = _shared_decode(g, dplan, 7)
    assert err == 0 and torch.equal(out, ref)


@pytest.mark.parametrize("G,max_group", [(1, 32), (2, 16), (4, 8), (5, 6), (8, 4)])
@pytest.mark.parametrize("BS", [16, 32])
def test_group_shapes(G, max_group, BS):
    """Every query-group size with as many members as 32 columns hold; ragged lengths, shared
    prefixes of different depths, members whose last shared block ends their sequence."""
    Hkv = 2
    rng = np.random.default_rng(100 * G + BS)
    lengths = [int(x) for x in rng.integers(1, 12 * BS, size=2 * max_group + 3)]
    lengths[0] = 4 * BS                                  # a member whose every block is shared
    spec = W.Spec(f"pfx_{G}_{BS}", len(lengths), G * Hkv, Hkv, 128, BS, "bf16", "bf16", "bf16",
                  ("list", tuple(lengths)), ("fixed", 4 * sum(-(-L // BS) for L in lengths) + 8),
                  share_group=max_group, share_blocks=6, max_blocks_per_seq=12, seed=5000 + G * 10 + BS)
    b = W.build_batch(spec)
    ref, _, _ = oracle.run_step(b)
    g = GpuStep(b)
    g.append()
    plan, dplan = _plan(b, max_group)
    assert plan.num_groups >= 1
    for parts in (0, 5):
        out, err = _shared_decode(g, dplan, parts)
        assert err == 0
        assert max_err(out, ref) <= TOL["bf16"], parts


def test_fork_tree_from_the_block_manager():
    """Tables from the host block manager: prompts forked into children that share whole blocks
    with their parent (and each other) to different depths, then decode steps."""
    Hq, Hkv, D, BS, NB = 8, 2, 128, 16, 512
    bm = blocks.BlockManager(NB, BS, 64)
    rng = np.random.default_rng(11)
    ids = []
    for p in range(3):                                   # three prompts, each forked into 4 children
        pid = 100 * p
        assert bm.add(pid, int(rng.integers(40, 200))) == 0
        ids.append(pid)
        for c in range(1, 5):
            assert bm.fork(pid, pid + c) == 0
            ids.append(pid + c)
            for _ in range(int(rng.integers(0, 40))):    # children drift apart
                assert bm.append(pid + c)[0] == 0
    st, slots, tables, lens, cows, n_done = bm.step(ids)
    assert st == 0 and n_done == len(ids)
    S = len(ids)
    spec = W.Spec("fork_tree", S, Hq, Hkv, D, BS, "bf16", "bf16", "bf16", ("list", tuple(int(x) for x in lens)),
                  ("fixed", NB), max_blocks_per_seq=64, seed=77)
    b = W.batch_from_tables(spec, tables, lens, NB)
    ref, _, _ = oracle.run_step(b)
    g = GpuStep(b)
    g.append()
    plan, dplan = _plan(b, 8)
    assert plan.num_groups >= 3
    out, err = _shared_decode(g, dplan, 0)
    assert err == 0
    assert max_err(out, ref) <= TOL["bf16"]


def test_bad_plan_is_flagged_not_faulted():
    """A shared count beyond a sequence's full blocks sets PKV_DEVERR_PLAN; nothing faults."""
    b = W.config_batch(3, num_seqs=16)
    g = GpuStep(b)
    g.append()
    plan, _ = _plan(b, 8)
    s = int(np.argmax(plan.shared))
    plan.shared[s] = int(b.seq_lens[s]) // b.spec.block_size + 3
    _, err = _shared_decode(g, pkv.DevicePrefixPlan(plan, 8), 0)
    assert err & pkv.DEVERR_PLAN
