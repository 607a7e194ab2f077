"""CUDA path against the CPU oracle, element by element, through the C ABI.

Tolerances (max |gpu - oracle| over every output element, oracle in fp64 on the
same rounded inputs): 1e-5 for fp32 caches, 1e-2 for bf16, 3e-2 for FP8-E4M3.
The append (reshape_and_cache) must be bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_462_b200 as pkv
import workloads as W
from gpu_harness import TOL, TORCH_DT, GpuStep, cache_bytes, max_err, to_dev, to_f64

pytestmark = pytest.mark.gpu


def _spec(name, S, Hq, Hkv, D, BS, kv, lengths, pool=None, seed=1, share=0):
    q = "f32" if kv == "f32" else "bf16"
    nb = max(1, -(-max(lengths) // BS))
    pool = pool or ("fixed", max(8, 2 * sum(-(-L // BS) for L in lengths) + 3))
    return W.Spec(name, S, Hq, Hkv, D, BS, q, q, kv, ("list", tuple(lengths)), pool,
                  share_group=share, share_blocks=4 if share else 0, max_blocks_per_seq=nb + 1, seed=seed)


def _check_step(batch, partitions=(0,)):
    ref, okc, ovc = oracle.run_step(batch)
    g = GpuStep(batch)
    g.append()
    torch.cuda.synchronize()
    assert np.array_equal(cache_bytes(g.kc), okc), "K cache differs from the oracle's append"
    assert np.array_equal(cache_bytes(g.vc), ovc), "V cache differs from the oracle's append"
    for parts in partitions:
        out = g.decode(parts)
        e = max_err(out, ref)
        assert e <= TOL[batch.spec.kv_dtype], (parts, e)
        assert g.device_errors() == 0
    return g, ref


# ------------------------------------------------------------------ append

def test_append_fp8_special_values():
    """Saturation, ties, subnormals and signed zero through the hardware E4M3 conversion."""
    vals = np.array([0.0, -0.0, 448.0, 449.0, 1e9, -1e9, np.inf, -np.inf, 2.0 ** -10, -(2.0 ** -10),
                     3 * 2.0 ** -11, 1.0625, 1.1875, 17.0, 19.0, 240.0, 248.0, 2.0 ** -9, 1e-30, 0.3],
                    dtype=np.float32)
    D = 64
    rows = np.resize(vals, (3, 1, D)).astype(np.float32)
    rows[1] *= -1.5
    rows[2] = np.random.default_rng(3).standard_normal((1, D)).astype(np.float32) * 1000
    slots = np.array([3, 17, 40], np.int64)
    okc = oracle.empty_cache(4, 1, 16, D, "e4m3"); ovc = oracle.empty_cache(4, 1, 16, D, "e4m3")
    oracle.reshape_and_cache(rows, rows, "f32", okc, ovc, "e4m3", slots, 1, D, 16, 4, 1.0, 0.5)
    kc = torch.zeros(4, 1, 16, D, dtype=torch.uint8, device="cuda"); vc = torch.zeros_like(kc)
    t = torch.from_numpy(rows).cuda()
    pkv.reshape_and_cache(t, t.clone(), kc, vc, torch.from_numpy(slots).cuda(), 1.0, 0.5)
    assert np.array_equal(kc.cpu().numpy(), okc)
    assert np.array_equal(vc.cpu().numpy(), ovc)


@pytest.mark.parametrize("kv,inp", [("f32", "f32"), ("bf16", "bf16"), ("e4m3", "bf16"), ("e4m3", "f32")])
def test_append_bit_exact_and_padding(kv, inp):
    rng = np.random.default_rng(5)
    T, Hkv, D, BS, NB = 300, 4, 128, 16, 40
    rows_k = rng.standard_normal((T, Hkv, D)).astype(np.float32) * 3
    rows_v = rng.standard_normal((T, Hkv, D)).astype(np.float32)
    if inp == "bf16":
        rows_k, rows_v = W.f32_to_bf16_bits(rows_k), W.f32_to_bf16_bits(rows_v)
    slots = rng.permutation(NB * BS)[:T].astype(np.int64)
    slots[::7] = -1                                          # padding rows write nothing
    ks, vs = (np.float32(3 * 4.5 / 448), np.float32(4.5 / 448)) if kv == "e4m3" else (np.float32(1), np.float32(1))
    okc = oracle.empty_cache(NB, Hkv, BS, D, kv); ovc = oracle.empty_cache(NB, Hkv, BS, D, kv)
    oracle.reshape_and_cache(rows_k, rows_v, inp, okc, ovc, kv, slots, Hkv, D, BS, NB, ks, vs)
    kc = torch.zeros(okc.shape, dtype={"f32": torch.float32, "bf16": torch.bfloat16, "e4m3": torch.uint8}[kv],
                     device="cuda")
    vc = torch.zeros_like(kc)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.reshape_and_cache(to_dev(rows_k, inp), to_dev(rows_v, inp), kc, vc, torch.from_numpy(slots).cuda(),
                          float(ks), float(vs), err)
    assert np.array_equal(cache_bytes(kc), okc) and np.array_equal(cache_bytes(vc), ovc)
    assert int(err.item()) == 0


def test_append_slot_past_pool_is_flagged_not_written():
    k = torch.ones(3, 2, 64, device="cuda")
    kc = torch.zeros(2, 2, 16, 64, device="cuda"); vc = torch.zeros_like(kc)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.reshape_and_cache(k, k, kc, vc, torch.tensor([1, 32, 5000], device="cuda"), device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == pkv.DEVERR_SLOT
    assert kc.sum().item() == 2 * 64 and kc[0, :, 1].eq(1).all()


# ------------------------------------------------------------------ decode

def test_config0_full():
    b = W.config_batch(0)
    _check_step(b, partitions=(0, 1, 2, 3, 7, 16, 1000))


@pytest.mark.parametrize("kv", ["f32", "bf16", "e4m3"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("BS", [8, 16, 32])
@pytest.mark.parametrize("G", [1, 2, 4, 5, 8])
def test_shapes_grid(kv, D, BS, G):
    Hkv = 2
    lengths = [0, 1, BS, BS + 1, 3 * BS - 1, 97, 200]
    b = W.build_batch(_spec(f"grid_{kv}_{D}_{BS}_{G}", len(lengths), G * Hkv, Hkv, D, BS, kv, lengths,
                            seed=D * 1000 + BS * 10 + G))
    g, _ = _check_step(b, partitions=(0, 5))
    out = g.out.float().cpu().numpy()
    assert np.all(out[0] == 0)                               # empty sequence: zero row


@pytest.mark.parametrize("cfg", [1, 2, 3, 4])
def test_configs_cut_down_every_output(cfg):
    """Same distributions as the full workloads, a few sequences: every output element checked."""
    over = {1: dict(num_seqs=6), 2: dict(num_seqs=2, lengths=("fixed", 2000)),
            3: dict(num_seqs=16), 4: dict(num_seqs=5)}[cfg]
    b = W.config_batch(cfg, **over)
    _check_step(b, partitions=(0, 1, 3, 17, 148))


def test_split_invariance_sweep():
    b = W.config_batch(1, num_seqs=8)
    ref, _, _ = oracle.run_step(b)
    g = GpuStep(b)
    g.append()
    for parts in (1, 2, 3, 4, 5, 8, 13, 16, 37, 64, 148, 296, 592, 2000):
        e = max_err(g.decode(parts), ref)
        assert e <= TOL["bf16"], (parts, e)
    assert g.device_errors() == 0


@pytest.mark.parametrize("cfg,kv", [(1, None), (2, None), (3, None), (4, None), (2, "e4m3"), (3, "e4m3")])
def test_full_size_sampled(cfg, kv, fp8_kernel):
    """Full workload in the benchmark's launch configuration; sampled sequences checked one by one."""
    if fp8_kernel == "tcgen05" and (kv or W.config_spec(cfg).kv_dtype) not in ("e4m3", "e5m2"):
        pytest.skip("the FP8 kernel choice only concerns FP8 caches")
    b = W.config_batch(cfg) if kv is None else W.with_cache_dtype(W.config_batch(cfg), kv)
    g = GpuStep(b)
    out = g.step(0)
    torch.cuda.synchronize()
    assert g.device_errors() == 0
    assert torch.isfinite(out.float()).all()
    rng = np.random.default_rng(cfg)
    seqs = sorted(set(rng.choice(b.num_seqs, size=min(6, b.num_seqs), replace=False).tolist())
                  | {int(np.argmax(b.seq_lens)), int(np.argmin(b.seq_lens))})
    ref, okc, ovc = oracle.run_step(b, seqs=seqs)
    e = max_err(out, ref, seqs)
    assert e <= TOL[b.spec.kv_dtype], e
    # every block those sequences read (history fill + the step's append) is bit-exact
    bs = b.spec.block_size
    nb = b.nblocks()
    blocks = np.unique(np.concatenate([b.block_tables[s, :nb[s]] for s in seqs]))
    idx = torch.from_numpy(blocks.astype(np.int64)).cuda()
    assert np.array_equal(cache_bytes(g.kc[idx]), okc[blocks])
    assert np.array_equal(cache_bytes(g.vc[idx]), ovc[blocks])


def test_prefix_sharing_equals_private_copies():
    """Shared prefix blocks are read-only reuse: duplicating them physically changes nothing."""
    b = W.config_batch(3, num_seqs=16)
    g1 = GpuStep(b)
    o1 = g1.step(7).clone()
    # private copy of every shared block, appended to the pool
    bs = b.spec.block_size
    nb = b.nblocks()
    used = {}
    tables = b.block_tables.copy()
    extra_src = []
    for s in range(b.num_seqs):
        for j in range(nb[s]):
            p = int(tables[s, j])
            if p in used:
                tables[s, j] = b.num_blocks + len(extra_src)
                extra_src.append(p)
            used.setdefault(p, s)
    assert extra_src, "workload has no shared blocks"
    g2 = GpuStep(b)
    g2.append()
    kc2 = torch.cat([g2.kc, g2.kc[torch.tensor(extra_src, device="cuda")]])
    vc2 = torch.cat([g2.vc, g2.vc[torch.tensor(extra_src, device="cuda")]])
    out2 = torch.empty_like(g2.q)
    ws = pkv.new_workspace(b.num_seqs, b.spec.num_heads, b.spec.num_kv_heads, b.spec.head_dim, 7)
    pkv.paged_attention_decode(out2, g2.q, kc2, vc2, torch.from_numpy(tables).cuda(), g2.sl, float(b.scale),
                               num_partitions=7, workspace=ws)
    assert torch.equal(o1, out2)


def test_permutation_invariance_bit_exact():
    b = W.config_batch(1, num_seqs=8)
    g = GpuStep(b)
    o1 = g.step(11).clone()
    perm = torch.from_numpy(np.random.default_rng(9).permutation(b.num_blocks)).cuda()
    kc2 = torch.empty_like(g.kc); vc2 = torch.empty_like(g.vc)
    kc2[perm] = g.kc; vc2[perm] = g.vc
    bt = torch.from_numpy(b.block_tables).cuda()
    bt2 = torch.where(bt >= 0, perm[bt.clamp(min=0).long()].int(), bt)
    out2 = torch.empty_like(g.q)
    pkv.paged_attention_decode(out2, g.q, kc2, vc2, bt2, g.sl, float(b.scale), num_partitions=11,
                               workspace=pkv.new_workspace(8, 32, 8, 128, 11))
    assert torch.equal(o1, out2)


def test_bad_block_id_is_flagged_and_skipped():
    b = W.config_batch(1, num_seqs=4)
    g = GpuStep(b)
    g.append()
    bt = b.block_tables.copy()
    bt[2, 3] = b.num_blocks + 5                              # outside the pool
    g.bt = torch.from_numpy(bt).cuda()
    out = g.decode(0)
    torch.cuda.synchronize()
    assert g.device_errors() & pkv.DEVERR_BLOCK_ID
    ref, _, _ = oracle.run_step(b, seqs=[0, 1, 3])
    assert max_err(out, ref, [0, 1, 3]) <= TOL["bf16"]       # other sequences untouched


def test_bad_seq_len_is_flagged_and_clamped():
    b = W.config_batch(0)
    g = GpuStep(b)
    g.append()
    sl = b.seq_lens.copy()
    sl[1] = 10_000                                           # beyond max_blocks_per_seq * block_size
    g.sl = torch.from_numpy(sl).cuda()
    g.decode(0)
    assert g.device_errors() & pkv.DEVERR_SEQ_LEN


# ------------------------------------------------------------------ fused step

@pytest.mark.parametrize("cfg,over", [(0, {}), (1, dict(num_seqs=8)), (3, dict(num_seqs=16)), (4, dict(num_seqs=6)),
                                      (2, dict(num_seqs=2, lengths=("fixed", 1000)))])
@pytest.mark.parametrize("parts", [0, 3, 64])
def test_fused_step_matches_oracle_and_two_calls(cfg, over, parts):
    """paged_decode_step = reshape_and_cache + paged_attention_decode: same caches (bit-exact),
    outputs within tolerance of the oracle and identical to the two separate calls."""
    b = W.config_batch(cfg, **over)
    ref, okc, ovc = oracle.run_step(b)
    g1 = GpuStep(b)
    out1 = g1.fused_step(parts).clone()
    assert g1.device_errors() == 0
    assert np.array_equal(cache_bytes(g1.kc), okc) and np.array_equal(cache_bytes(g1.vc), ovc)
    assert max_err(out1, ref) <= TOL[b.spec.kv_dtype]
    g2 = GpuStep(b)
    out2 = g2.step(parts)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2)


@pytest.mark.parametrize("kv", ["bf16", "e4m3"])
@pytest.mark.parametrize("BS", [8, 16, 32])
def test_fused_step_shapes(kv, BS):
    lengths = [1, BS, BS + 1, 3 * BS - 1, 97, 200, 0]
    b = W.build_batch(_spec(f"fused_{kv}_{BS}", len(lengths), 8, 2, 128, BS, kv, lengths, seed=77 + BS))
    ref, okc, ovc = oracle.run_step(b)
    g = GpuStep(b)
    out = g.fused_step(5)
    assert g.device_errors() == 0
    assert np.array_equal(cache_bytes(g.kc), okc) and np.array_equal(cache_bytes(g.vc), ovc)
    assert max_err(out, ref) <= TOL[kv]


def test_fused_step_negative_slot_appends_nothing():
    """A negative slot skips that sequence's append; its decode then reads the (zero) row."""
    b = W.config_batch(1, num_seqs=6)
    b.new_slots[[1, 4]] = -1
    ref, okc, ovc = oracle.run_step(b)
    g = GpuStep(b)
    out = g.fused_step(0)
    assert g.device_errors() == 0
    assert np.array_equal(cache_bytes(g.kc), okc) and np.array_equal(cache_bytes(g.vc), ovc)
    assert max_err(out, ref) <= TOL["bf16"]


def test_fused_step_flags_slot_outside_last_block():
    b = W.config_batch(1, num_seqs=4)
    g = GpuStep(b)
    slots = b.new_slots.copy()
    slots[2] = int(b.block_tables[2, 0]) * b.spec.block_size    # first block, not the last
    g.new_slots = torch.from_numpy(slots).cuda()
    out = g.fused_step(0)
    assert g.device_errors() & pkv.DEVERR_SLOT
    ref, _, _ = oracle.run_step(b, seqs=[0, 1, 3])
    assert max_err(out, ref, [0, 1, 3]) <= TOL["bf16"]           # other sequences untouched


def test_fused_step_flags_slot_of_empty_sequence():
    lengths = [40, 0, 17]
    b = W.build_batch(_spec("fused_empty_slot", len(lengths), 8, 2, 128, 16, "bf16", lengths, seed=5))
    g = GpuStep(b)
    slots = b.new_slots.copy()
    slots[1] = 0
    g.new_slots = torch.from_numpy(slots).cuda()
    out = g.fused_step(0)
    assert g.device_errors() & pkv.DEVERR_SLOT
    assert not torch.any(out[1].float() != 0)


def test_bounded_wait_runs_out_and_context_survives():
    """Failure path: a stage that never fills makes the consumers' bounded wait run out (~1 s);
    the launch returns with DEVERR_TIMEOUT in the workspace and the context keeps working."""
    b = W.config_batch(1, num_seqs=8)
    g = GpuStep(b)
    g.append()
    ws = pkv.new_workspace(b.num_seqs, b.spec.num_heads, b.spec.num_kv_heads, b.spec.head_dim, 0)
    pkv.withheld_unit_decode(g.out, g.q, g.kc, g.vc, g.bt, g.sl, float(b.scale), 5, ws)
    torch.cuda.synchronize()
    assert pkv.read_device_error(ws) & pkv.DEVERR_TIMEOUT
    with pytest.raises(pkv.PkvError):
        pkv.withheld_unit_decode(g.out, g.q, g.kc, g.vc, g.bt, g.sl, float(b.scale), -1, ws)
    pkv.workspace_init(ws)
    out = g.decode(0, ws)
    torch.cuda.synchronize()
    assert pkv.read_device_error(ws) == 0
    ref, _, _ = oracle.run_step(b)
    assert max_err(out, ref) <= TOL["bf16"]


@pytest.mark.parametrize("cfg", [1, 4])
@pytest.mark.parametrize("parts", [0, 7])
def test_guard_regions_untouched(cfg, parts):
    """Canaries before and after `out` and after the workspace survive a fused step."""
    b = W.config_batch(cfg, num_seqs=6)
    sp = b.spec
    g = GpuStep(b)
    guard = 4096
    n = g.out.numel()
    big = torch.empty(guard + n + guard, dtype=g.out.dtype, device=g.out.device)
    big.view(torch.int16).fill_(0x7FC1)                      # a NaN pattern no result takes
    g.out = big[guard:guard + n].view_as(g.q)
    wbytes = pkv.workspace_size(b.num_seqs, sp.num_heads, sp.num_kv_heads, sp.head_dim, parts)
    wbig = torch.zeros(wbytes + 65536, dtype=torch.uint8, device=g.out.device)
    wbig[wbytes:].fill_(0xA5)
    ws = wbig[:wbytes]
    pkv.workspace_init(ws)
    g.fused_step(parts, ws)
    torch.cuda.synchronize()
    assert pkv.read_device_error(ws) == 0
    assert bool((big[:guard].view(torch.int16) == 0x7FC1).all()) and bool((big[guard + n:].view(torch.int16) == 0x7FC1).all())
    assert bool((wbig[wbytes:] == 0xA5).all())
    ref, _, _ = oracle.run_step(b)
    assert max_err(g.out, ref) <= TOL[sp.kv_dtype]


# ------------------------------------------------------------------ E5M2 caches

def test_append_e5m2_special_values():
    """Saturation at 57344, ties, subnormals, signed zero through the hardware E5M2 conversion;
    NaN inputs must give a NaN code (which NaN code is not fixed by the format)."""
    vals = np.array([0.0, -0.0, 57344.0, 60000.0, 61440.0, 1e9, -1e9, np.inf, -np.inf, 2.0 ** -16, -(2.0 ** -17),
                     3 * 2.0 ** -18, 1.125, 1.375, 20.0, 28.0, 12288.0, 2.0 ** -14, 1e-30, 0.3, np.nan],
                    dtype=np.float32)
    D = 64
    rows = np.resize(vals, (3, 1, D)).astype(np.float32)
    rows[1] *= -1.5
    rows[2] = np.random.default_rng(4).standard_normal((1, D)).astype(np.float32) * 1000
    slots = np.array([3, 17, 40], np.int64)
    okc = oracle.empty_cache(4, 1, 16, D, "e5m2"); ovc = oracle.empty_cache(4, 1, 16, D, "e5m2")
    oracle.reshape_and_cache(rows, rows, "f32", okc, ovc, "e5m2", slots, 1, D, 16, 4, 1.0, 0.5)
    kc = torch.zeros(4, 1, 16, D, dtype=torch.float8_e5m2, device="cuda"); vc = torch.zeros_like(kc)
    t = torch.from_numpy(rows).cuda()
    pkv.reshape_and_cache(t, t.clone(), kc, vc, torch.from_numpy(slots).cuda(), 1.0, 0.5)
    for got, ref in ((cache_bytes(kc), okc), (cache_bytes(vc), ovc)):
        nan_ref = (ref & 0x7C) == 0x7C
        nan_ref &= (ref & 0x03) != 0
        nan_got = ((got & 0x7C) == 0x7C) & ((got & 0x03) != 0)
        assert np.array_equal(nan_ref, nan_got)
        assert np.array_equal(got[~nan_ref], ref[~nan_ref])


@pytest.mark.parametrize("inp", ["bf16", "f32"])
def test_append_e5m2_bit_exact(inp):
    rng = np.random.default_rng(6)
    T, Hkv, D, BS, NB = 300, 4, 128, 16, 40
    rows_k = rng.standard_normal((T, Hkv, D)).astype(np.float32) * 3
    rows_v = rng.standard_normal((T, Hkv, D)).astype(np.float32)
    if inp == "bf16":
        rows_k, rows_v = W.f32_to_bf16_bits(rows_k), W.f32_to_bf16_bits(rows_v)
    slots = rng.permutation(NB * BS)[:T].astype(np.int64)
    slots[::7] = -1
    ks, vs = np.float32(3 * 4.5 / 57344), np.float32(4.5 / 57344)
    okc = oracle.empty_cache(NB, Hkv, BS, D, "e5m2"); ovc = oracle.empty_cache(NB, Hkv, BS, D, "e5m2")
    oracle.reshape_and_cache(rows_k, rows_v, inp, okc, ovc, "e5m2", slots, Hkv, D, BS, NB, ks, vs)
    kc = torch.zeros(okc.shape, dtype=torch.float8_e5m2, device="cuda"); vc = torch.zeros_like(kc)
    pkv.reshape_and_cache(to_dev(rows_k, inp), to_dev(rows_v, inp), kc, vc, torch.from_numpy(slots).cuda(),
                          float(ks), float(vs))
    assert np.array_equal(cache_bytes(kc), okc) and np.array_equal(cache_bytes(vc), ovc)


@pytest.mark.parametrize("BS", [16, 32])
@pytest.mark.parametrize("G", [1, 2, 4, 5, 8])
def test_e5m2_shapes(BS, G):
    Hkv = 2
    lengths = [0, 1, BS, BS + 1, 3 * BS - 1, 97, 200]
    b = W.build_batch(_spec(f"e5m2_{BS}_{G}", len(lengths), G * Hkv, Hkv, 128, BS, "e5m2", lengths,
                            seed=5000 + BS * 10 + G))
    g, _ = _check_step(b, partitions=(0, 5))
    assert np.all(g.out.float().cpu().numpy()[0] == 0)


@pytest.fixture
def tcgen05():
    """FP8-cache decodes on the tcgen05 kernel for the test, the default kernel after it."""
    prev = pkv.set_fp8_kernel(pkv.FP8_KERNEL_TCGEN05)
    yield
    pkv.set_fp8_kernel(prev)


@pytest.fixture(params=["mma", "tcgen05"])
def fp8_kernel(request):
    """Both FP8-cache kernels in turn."""
    prev = pkv.set_fp8_kernel(pkv.FP8_KERNEL_TCGEN05 if request.param == "tcgen05" else pkv.FP8_KERNEL_MMA)
    yield request.param
    pkv.set_fp8_kernel(prev)


@pytest.mark.parametrize("kv", ["e4m3", "e5m2"])
@pytest.mark.parametrize("BS", [16, 32])
@pytest.mark.parametrize("G", [1, 2, 4, 5, 8])
def test_fp8_tensor_core_shapes(kv, BS, G, fp8_kernel):
    """FP8 caches whose KV heads fill whole 128-row tiles (128 / block_size heads of a block per
    unit, one and two head groups): ragged lengths, one and several partitions (streams split
    across CTAs and merged), every output element against the oracle."""
    hpu = 128 // BS
    for Hkv in (hpu, 2 * hpu):
        lengths = [0, 1, BS, BS + 1, 3 * BS - 1, 97, 200, 700]
        b = W.build_batch(_spec(f"tc_{kv}_{BS}_{G}_{Hkv}", len(lengths), G * Hkv, Hkv, 128, BS, kv, lengths,
                                seed=7000 + BS * 10 + G + Hkv))
        g, _ = _check_step(b, partitions=(0, 5, 40))
        assert np.all(g.out.float().cpu().numpy()[0] == 0)


@pytest.mark.parametrize("cfg,over", [(1, dict(num_seqs=6)), (4, dict(num_seqs=5)), (3, dict(num_seqs=16)),
                                      (2, dict(num_seqs=2, lengths=("fixed", 2000)))])
def test_e5m2_workloads_fused_step(cfg, over, fp8_kernel):
    b = W.config_batch(cfg, kv_dtype="e5m2", **over)
    ref, okc, ovc = oracle.run_step(b)
    g = GpuStep(b)
    out = g.fused_step(0)
    assert g.device_errors() == 0
    assert np.array_equal(cache_bytes(g.kc), okc) and np.array_equal(cache_bytes(g.vc), ovc)
    assert max_err(out, ref) <= TOL["e5m2"]


def test_e5m2_uncovered_shapes_are_rejected():
    """E5M2 is decoded by the tensor-core kernel only: head_dim 64 or block 8 is refused before any launch."""
    for D, BS in ((64, 16), (128, 8)):
        q = torch.zeros(2, 4, D, dtype=torch.bfloat16, device="cuda")
        kc = torch.zeros(4, 2, BS, D, dtype=torch.float8_e5m2, device="cuda")
        bt = torch.zeros(2, 2, dtype=torch.int32, device="cuda")
        sl = torch.ones(2, dtype=torch.int32, device="cuda")
        with pytest.raises(pkv.PkvError):
            pkv.paged_attention_decode(torch.empty_like(q), q, kc, kc.clone(), bt, sl, 0.1, 1.0, 1.0)


# ------------------------------------------------------------------ several new tokens per sequence

@pytest.mark.parametrize("kv", ["bf16", "e4m3"])
@pytest.mark.parametrize("BS", [16, 32])
@pytest.mark.parametrize("q_len,Hq,Hkv", [(2, 8, 2), (4, 4, 2), (8, 2, 2), (2, 4, 2), (5, 2, 2)])
def test_multi_query_causal(kv, BS, q_len, Hq, Hkv):
    """q_len new tokens per sequence against the oracle's causal definition, every output element;
    lengths include sequences shorter than the chunk (their early queries see nothing)."""
    lengths = [1, q_len - 1 if q_len > 1 else 1, q_len, BS + 3, 3 * BS - 1, 97, 300]
    b = W.build_batch(_spec(f"mq_{kv}_{BS}_{q_len}_{Hq}", len(lengths), Hq, Hkv, 128, BS, kv, lengths,
                            seed=900 + BS + q_len * 10 + Hq))
    sp = b.spec
    _, okc, ovc = oracle.run_step(b)
    g = GpuStep(b)
    g.append()
    rng = np.random.default_rng(q_len * 100 + Hq)
    qm = W.f32_to_bf16_bits(rng.standard_normal((b.num_seqs, q_len, Hq, 128)).astype(np.float32))
    ref = oracle.paged_decode(qm, "bf16", okc, ovc, kv, b.block_tables, b.seq_lens, Hq, Hkv, 128, BS, b.num_blocks,
                              b.scale, b.k_scale, b.v_scale, q_len=q_len)
    q = to_dev(qm, "bf16")
    for parts in (0, 3):
        out = torch.full_like(q, float("nan"))
        ws = pkv.new_workspace(b.num_seqs, Hq * q_len, Hkv, 128, parts)
        pkv.paged_attention_decode_mq(out, q, g.kc, g.vc, g.bt, g.sl, float(b.scale), float(b.k_scale),
                                      float(b.v_scale), parts, ws)
        torch.cuda.synchronize()
        assert pkv.read_device_error(ws) == 0
        got = out.double().cpu().numpy()
        assert np.isfinite(got).all()
        assert np.max(np.abs(got - ref)) <= TOL[kv], parts


@pytest.mark.parametrize("kv", ["e4m3", "e5m2"])
@pytest.mark.parametrize("BS,q_len,Hq,Hkv", [(16, 2, 16, 8), (16, 4, 16, 8), (16, 5, 8, 8), (32, 2, 8, 4)])
def test_multi_query_causal_fp8_tensor_core(kv, BS, q_len, Hq, Hkv, fp8_kernel):
    """Several new tokens per sequence on FP8 caches whose heads fill whole 128-row tiles (the
    columns of a KV head are its query heads x new tokens), against the oracle's causal definition."""
    lengths = [1, q_len - 1, q_len, BS + 3, 3 * BS - 1, 97, 300]
    b = W.build_batch(_spec(f"mqtc_{kv}_{BS}_{q_len}_{Hq}", len(lengths), Hq, Hkv, 128, BS, kv, lengths,
                            seed=1900 + BS + q_len * 10 + Hq))
    _, okc, ovc = oracle.run_step(b)
    g = GpuStep(b)
    g.append()
    rng = np.random.default_rng(q_len * 100 + Hq + 7)
    qm = W.f32_to_bf16_bits(rng.standard_normal((b.num_seqs, q_len, Hq, 128)).astype(np.float32))
    ref = oracle.paged_decode(qm, "bf16", okc, ovc, kv, b.block_tables, b.seq_lens, Hq, Hkv, 128, BS, b.num_blocks,
                              b.scale, b.k_scale, b.v_scale, q_len=q_len)
    q = to_dev(qm, "bf16")
    for parts in (0, 3):
        out = torch.full_like(q, float("nan"))
        ws = pkv.new_workspace(b.num_seqs, Hq * q_len, Hkv, 128, parts)
        pkv.paged_attention_decode_mq(out, q, g.kc, g.vc, g.bt, g.sl, float(b.scale), float(b.k_scale),
                                      float(b.v_scale), parts, ws)
        torch.cuda.synchronize()
        assert pkv.read_device_error(ws) == 0
        got = out.double().cpu().numpy()
        assert np.isfinite(got).all()
        assert np.max(np.abs(got - ref)) <= TOL[kv], parts


def test_multi_query_one_token_is_decode():
    b = W.config_batch(1, num_seqs=6)
    g = GpuStep(b)
    g.append()
    out1 = g.decode(0).clone()
    out2 = torch.empty_like(out1)
    sp = b.spec
    ws = pkv.new_workspace(b.num_seqs, sp.num_heads, sp.num_kv_heads, sp.head_dim, 0)
    pkv.paged_attention_decode_mq(out2.view(b.num_seqs, 1, sp.num_heads, sp.head_dim),
                                  g.q.view(b.num_seqs, 1, sp.num_heads, sp.head_dim), g.kc, g.vc, g.bt, g.sl,
                                  float(b.scale), 1.0, 1.0, 0, ws)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2)


def test_multi_query_unsupported_shapes_are_rejected():
    q = torch.zeros(2, 3, 4, 128, dtype=torch.bfloat16, device="cuda")      # 3 tokens x G 2 = 6 columns
    kc = torch.zeros(8, 2, 16, 128, dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros(2, 2, dtype=torch.int32, device="cuda")
    sl = torch.full((2,), 5, dtype=torch.int32, device="cuda")
    with pytest.raises(pkv.PkvError):
        pkv.paged_attention_decode_mq(torch.empty_like(q), q, kc, kc.clone(), bt, sl, 0.1)


# ------------------------------------------------------------------ per-KV-head FP8 scales

def _head_scale_case(kv, parts, gain_k, gain_v):
    """Config 1 cut down with K and V rows of KV head h scaled by gain_k[h] / gain_v[h], 8-bit caches
    with per-head absmax scales: GPU and oracle caches and outputs (GPU output, oracle output)."""
    b = W.config_batch(1, num_seqs=6, kv_dtype=kv)
    sp = b.spec
    Hkv, D, BS, NB = sp.num_kv_heads, sp.head_dim, sp.block_size, b.num_blocks
    def rows(x, gain):
        f = W.bf16_bits_to_f32(x) * gain[None, :, None]
        return W.f32_to_bf16_bits(f.astype(np.float32))
    hk, nk = rows(b.hist_k, gain_k), rows(b.new_k, gain_k)
    hv, nv = rows(b.hist_v, gain_v), rows(b.new_v, gain_v)
    top = {"e4m3": 448.0, "e5m2": 57344.0, "int8": 127.0}[kv]
    def head_absmax(*xs):
        return np.max([np.abs(W.bf16_bits_to_f32(x)).max(axis=(0, 2)) for x in xs], axis=0)
    khs = (head_absmax(hk, nk) / np.float32(top)).astype(np.float32)
    vhs = (head_absmax(hv, nv) / np.float32(top)).astype(np.float32)
    okc = oracle.empty_cache(NB, Hkv, BS, D, kv); ovc = oracle.empty_cache(NB, Hkv, BS, D, kv)
    for k_, v_, sl_ in ((hk, hv, b.hist_slots), (nk, nv, b.new_slots)):
        oracle.reshape_and_cache(k_, v_, "bf16", okc, ovc, kv, sl_, Hkv, D, BS, NB,
                                 k_head_scales=khs, v_head_scales=vhs)
    ref = oracle.paged_decode(b.q, "bf16", okc, ovc, kv, b.block_tables, b.seq_lens, sp.num_heads, Hkv, D, BS, NB,
                              b.scale, k_head_scales=khs, v_head_scales=vhs)
    kc = torch.zeros((NB, Hkv, BS, D), dtype=TORCH_DT[kv], device="cuda"); vc = torch.zeros_like(kc)
    tk, tv = torch.from_numpy(khs).cuda(), torch.from_numpy(vhs).cuda()
    for k_, v_, sl_ in ((hk, hv, b.hist_slots), (nk, nv, b.new_slots)):
        pkv.reshape_and_cache_head_scales(to_dev(k_, "bf16"), to_dev(v_, "bf16"), kc, vc,
                                          torch.from_numpy(sl_).cuda(), tk, tv)
    out = torch.empty((b.num_seqs, sp.num_heads, D), dtype=torch.bfloat16, device="cuda")
    ws = pkv.new_workspace(b.num_seqs, sp.num_heads, Hkv, D, parts)
    pkv.paged_attention_decode_head_scales(out, to_dev(b.q, "bf16"), kc, vc, torch.from_numpy(b.block_tables).cuda(),
                                           torch.from_numpy(b.seq_lens).cuda(), float(b.scale), tk, tv, parts, ws)
    torch.cuda.synchronize()
    assert pkv.read_device_error(ws) == 0
    assert np.array_equal(cache_bytes(kc), okc) and np.array_equal(cache_bytes(vc), ovc)
    return to_f64(out), ref, sp.num_heads // Hkv


@pytest.mark.parametrize("kv", ["e4m3", "e5m2", "int8"])
@pytest.mark.parametrize("parts", [0, 5])
def test_head_scales_append_and_decode(kv, parts, fp8_kernel):
    """FP8 caches with one scale per KV head (heads of very different ranges): appends bit-exact
    and outputs within tolerance of the oracle using the same head scales, relative to each
    head's V range (outputs scale with it)."""
    gain = np.geomspace(0.05, 40.0, 8).astype(np.float32)           # per-head magnitude
    out, ref, G = _head_scale_case(kv, parts, gain, gain)
    err = np.abs(out - ref).max(axis=(0, 2))                          # per query head
    assert np.all(err <= TOL[kv] * np.repeat(gain, G)), err


@pytest.mark.parametrize("kv", ["e4m3", "e5m2", "int8"])
@pytest.mark.parametrize("parts", [0, 5])
def test_head_scales_unit_range_values_absolute_tolerance(kv, parts, fp8_kernel):
    """Per-head scales that differ widely for K (ranges 0.05x .. 40x) and moderately for V
    (0.5x .. 2x, values of order one): every output within the plain absolute tolerance."""
    gain_k = np.geomspace(0.05, 40.0, 8).astype(np.float32)
    gain_v = np.geomspace(0.5, 2.0, 8).astype(np.float32)[::-1].copy()
    out, ref, _ = _head_scale_case(kv, parts, gain_k, gain_v)
    assert np.abs(out - ref).max() <= TOL[kv]


@pytest.mark.parametrize("kv", ["e4m3", "e5m2", "int8"])
@pytest.mark.parametrize("qgain", [2.0 ** 8, 2.0 ** -16])
def test_8bit_cache_query_magnitudes(kv, qgain, fp8_kernel):
    """Queries far from unit size with 8-bit caches (q times 2^8: sharply peaked softmax; q times
    2^-16: nearly uniform): the fused step against the oracle on the same bf16 q."""
    b = W.config_batch(1, num_seqs=6, kv_dtype=kv)
    q = W.bf16_bits_to_f32(b.q) * np.float32(qgain)        # a power of two: exact in bf16
    b.q = W.f32_to_bf16_bits(q.astype(np.float32))
    ref, okc, ovc = oracle.run_step(b)
    g = GpuStep(b)
    out = g.fused_step(0)
    assert g.device_errors() == 0
    assert np.array_equal(cache_bytes(g.kc), okc) and np.array_equal(cache_bytes(g.vc), ovc)
    assert max_err(out, ref) <= TOL[kv]


# ------------------------------------------------------------------ INT8 caches

@pytest.mark.parametrize("inp", ["bf16", "f32"])
def test_append_int8_bit_exact(inp):
    rng = np.random.default_rng(7)
    T, Hkv, D, BS, NB = 300, 4, 128, 16, 40
    rows_k = rng.standard_normal((T, Hkv, D)).astype(np.float32) * 3
    rows_v = rng.standard_normal((T, Hkv, D)).astype(np.float32)
    if inp == "f32":                                        # ties, clamps, NaN and infinities too
        rows_k[0, 0, :12] = [0.5, 1.5, 2.5, -0.5, -2.5, 126.5, 127.5, 300.0, -300.0, np.nan, np.inf, -np.inf]
    if inp == "bf16":
        rows_k, rows_v = W.f32_to_bf16_bits(rows_k), W.f32_to_bf16_bits(rows_v)
    slots = rng.permutation(NB * BS)[:T].astype(np.int64)
    slots[::7] = -1
    slots[0] = 5
    ks = np.float32(1.0) if inp == "f32" else np.float32(3 * 4.5 / 127)
    vs = np.float32(4.5 / 127)
    okc = oracle.empty_cache(NB, Hkv, BS, D, "int8"); ovc = oracle.empty_cache(NB, Hkv, BS, D, "int8")
    oracle.reshape_and_cache(rows_k, rows_v, inp, okc, ovc, "int8", slots, Hkv, D, BS, NB, ks, vs)
    kc = torch.zeros(okc.shape, dtype=torch.int8, device="cuda"); vc = torch.zeros_like(kc)
    pkv.reshape_and_cache(to_dev(rows_k, inp), to_dev(rows_v, inp), kc, vc, torch.from_numpy(slots).cuda(),
                          float(ks), float(vs))
    assert np.array_equal(cache_bytes(kc), okc) and np.array_equal(cache_bytes(vc), ovc)


@pytest.mark.parametrize("BS", [16, 32])
@pytest.mark.parametrize("G", [1, 4, 5, 8])
def test_int8_shapes(BS, G):
    Hkv = 2
    lengths = [0, 1, BS, BS + 1, 3 * BS - 1, 97, 200]
    b = W.build_batch(_spec(f"int8_{BS}_{G}", len(lengths), G * Hkv, Hkv, 128, BS, "int8", lengths,
                            seed=7000 + BS * 10 + G))
    g, _ = _check_step(b, partitions=(0, 5))
    assert np.all(g.out.float().cpu().numpy()[0] == 0)


@pytest.mark.parametrize("cfg,over", [(1, dict(num_seqs=6)), (4, dict(num_seqs=5)), (3, dict(num_seqs=16))])
def test_int8_workloads_fused_step(cfg, over):
    b = W.config_batch(cfg, kv_dtype="int8", **over)
    ref, okc, ovc = oracle.run_step(b)
    g = GpuStep(b)
    out = g.fused_step(0)
    assert g.device_errors() == 0
    assert np.array_equal(cache_bytes(g.kc), okc) and np.array_equal(cache_bytes(g.vc), ovc)
    assert max_err(out, ref) <= TOL["int8"]


@pytest.mark.parametrize("kv", ["e4m3", "e5m2", "int8"])
@pytest.mark.parametrize("Hkv", [2, 8])
def test_every_8bit_code_reads_back_exactly(kv, Hkv, fp8_kernel):
    """One cached token (softmax weight exactly 1) whose V rows hold every finite code of the
    format across two KV heads: with a unit scale the output row is each code's value, bit for
    bit in bf16 (all of them are bf16 values): the kernel's use of each code is exact."""
    D, BS = 128, 16
    codes = np.arange(256, dtype=np.uint8)
    if kv == "e4m3":
        vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    elif kv == "e5m2":
        vals = torch.from_numpy(codes).view(torch.float8_e5m2).float().numpy()
    else:
        vals = codes.view(np.int8).astype(np.float32)
    bad = ~np.isfinite(vals)
    codes[bad], vals[bad] = 0, 0.0                          # NaN / infinite codes are not values
    kc = torch.zeros((4, Hkv, BS, D), dtype=TORCH_DT[kv], device="cuda")
    vc = torch.zeros_like(kc)
    vc.view(torch.uint8)[0, :2, 0, :] = torch.from_numpy(codes.reshape(2, D)).cuda()
    q = torch.ones((1, Hkv, D), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    pkv.paged_attention_decode(out, q, kc, vc, torch.zeros((1, 1), dtype=torch.int32, device="cuda"),
                               torch.ones(1, dtype=torch.int32, device="cuda"), 0.1, 1.0, 1.0)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy()
    assert np.array_equal(got[0, :2].reshape(-1), vals)
    assert np.all(got[0, 2:] == 0)
