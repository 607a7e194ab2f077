"""The seeded input generator: determinism and the structure the workloads promise."""
import numpy as np
import pytest

import workloads as W


def test_bf16_rounding_matches_torch():
    import torch
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100_000).astype(np.float32) * 10,
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5 - 2 ** -7], np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(W.f32_to_bf16_bits(x), ref)
    assert np.array_equal(W.bf16_bits_to_f32(ref), torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).float().numpy())


@pytest.mark.parametrize("cfg", [0, 1, 4])
def test_deterministic(cfg):
    kw = {} if cfg == 0 else {"num_seqs": 3}
    a, b = W.config_batch(cfg, **kw), W.config_batch(cfg, **kw)
    for f in ("seq_lens", "block_tables", "q", "hist_k", "hist_v", "hist_slots", "new_k", "new_slots"):
        assert np.array_equal(getattr(a, f), getattr(b, f)), f


def _check_structure(b):
    sp = b.spec
    nb = b.nblocks()
    assert b.block_tables.shape == (sp.num_seqs, b.max_blocks_per_seq)
    for s in range(sp.num_seqs):
        row = b.block_tables[s]
        assert np.all((row[:nb[s]] >= 0) & (row[:nb[s]] < b.num_blocks))
        assert np.all(row[nb[s]:] == -1)
    # every referenced slot is written exactly once by the history fill
    assert np.unique(b.hist_slots).size == b.hist_slots.size
    assert b.hist_slots.size == b.unique_blocks() * sp.block_size
    # appends: one per sequence, unique, at logical position L - 1
    live = b.new_slots[b.seq_lens > 0]
    assert np.unique(live).size == live.size
    for s in range(sp.num_seqs):
        L = int(b.seq_lens[s])
        if L:
            assert b.new_slots[s] == b.block_tables[s, (L - 1) // sp.block_size] * sp.block_size + (L - 1) % sp.block_size


def test_config0_shape():
    b = W.config_batch(0)
    assert b.q.shape == (4, 8, 64) and b.q.dtype == np.float32
    assert b.num_blocks == 32 and np.all((b.seq_lens >= 1) & (b.seq_lens <= 64))
    _check_structure(b)


def test_config3_prefix_sharing_small():
    b = W.config_batch(3, num_seqs=16)
    _check_structure(b)
    sp = b.spec
    nb = b.nblocks()
    for g0 in range(0, 16, 8):
        for s in range(g0, g0 + 8):
            n = min(64, (int(b.seq_lens[s]) - 1) // 16)
            # shared prefix: identical to the group's longest-prefix member
            lead = max(range(g0, g0 + 8), key=lambda r: min(64, (int(b.seq_lens[r]) - 1) // 16))
            assert np.array_equal(b.block_tables[s, :n], b.block_tables[lead, :n])
            # private remainder: referenced by nobody else
            others = np.concatenate([b.block_tables[r, :nb[r]] for r in range(16) if r != s])
            assert not np.isin(b.block_tables[s, n:nb[s]], others).any()
    assert b.num_blocks % 1024 == 0 and b.num_blocks >= 2 * b.unique_blocks()


def test_config3_length_distribution():
    rng = np.random.default_rng(W.config_spec(3).seed)
    L = W._draw_lengths(W.config_spec(3), rng)
    assert L.size == 256 and L.min() >= 100 and L.max() <= 12000
    assert 1800 < np.median(L) < 2900


def test_fp8_scales_map_absmax_to_448():
    b = W.config_batch(4, num_seqs=2)
    assert b.hist_k.dtype == np.uint16
    absk = max(np.abs(W.bf16_bits_to_f32(b.hist_k)).max(), np.abs(W.bf16_bits_to_f32(b.new_k)).max())
    assert b.k_scale == np.float32(absk / np.float32(448))
    _check_structure(b)


def test_batch_layout_is_build_batch_tables():
    """The tables-only draw gives exactly the lengths, tables and pool of the full batch."""
    import workloads as W
    for i, kw in ((0, {}), (3, dict(num_seqs=24)), (1, dict(num_seqs=5))):
        b = W.config_batch(i, **kw)
        lay = W.batch_layout(b.spec)
        assert np.array_equal(lay.seq_lens, b.seq_lens) and np.array_equal(lay.block_tables, b.block_tables)
        assert lay.num_blocks == b.num_blocks


@pytest.mark.parametrize("kv", ["e4m3", "e5m2", "int8"])
def test_with_cache_dtype_equals_a_fresh_draw(kv):
    """Re-typing a drawn batch gives exactly what build_batch draws with the cache dtype replaced."""
    spec = W.config_spec(1)
    spec.num_seqs = 6
    a = W.with_cache_dtype(W.build_batch(spec), kv)
    spec.kv_dtype = kv
    b = W.build_batch(spec)
    assert a.spec.kv_dtype == kv and a.k_scale == b.k_scale and a.v_scale == b.v_scale
    for f in ("seq_lens", "block_tables", "q", "hist_k", "hist_v", "hist_slots", "new_k", "new_v", "new_slots"):
        assert np.array_equal(getattr(a, f), getattr(b, f)), f
