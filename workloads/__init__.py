"""Seeded synthetic decode batches for paged KV-cache attention.

This module only draws inputs: sequence lengths, block tables (a seeded
permutation of the physical pool, with whole prefix blocks shared inside a
group when asked), query / key / value tensors and the slot mapping of the
decode-step append. It holds none of the attention or cache arithmetic, so
both the CUDA library and the CPU oracle can be fed from it.

Workload shapes follow the pages' own examples:

* Llama-3-8B-like layer: 32 query heads, 8 KV heads, head_dim 128, bf16,
  block size 16 ("vLLM inference cost optimisation" article on
  developer.aliyun.com, section 2.1 "why the KV cache eats memory", and the
  wzjinhao.cn vLLM deployment write-up, section 2.1 PagedAttention).
* request lengths that differ widely (900 / 2300 / 4096 / 12000 tokens in the
  Aliyun article, section 3 "why traditional KV cache management is
  inefficient"), modelled as a log-normal with median 2300.
* prefix caching reuses whole blocks only (wzjinhao.cn write-up, section 2.3
  "Chunked Prefill and Prefix Caching").
* Qwen2.5-14B-like layer with an FP8 KV cache: 40 query heads, 8 KV heads
  (the wzjinhao.cn write-up's test model, section 3.3, with KV-cache FP8).

Conventions (a reading where the pages are silent):

* ``seq_lens[s]`` counts the token being decoded; that token sits at logical
  position ``L - 1`` and is written by the step's append (``new_k``/``new_v``
  at ``new_slots``). Every other referenced slot is written beforehand by the
  history fill (``hist_k``/``hist_v`` at ``hist_slots``), one row per slot of
  every referenced physical block.
* block-table rows are padded with -1 past ``ceil(L / block_size)``.
* bf16 tensors are returned as their uint16 bit patterns (round to nearest
  even from float32 draws); float32 tensors as float32.
"""
from __future__ import annotations

from dataclasses import dataclass, field
import math

import numpy as np

BASE_SEED = 462_000

DTYPES = ("f32", "bf16", "e4m3", "e5m2", "int8")


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return the bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    out = np.empty(u.shape, dtype=np.uint16)
    flat_u = u.reshape(-1)
    flat_o = out.reshape(-1)
    step = 1 << 24
    for i in range(0, flat_u.size, step):
        c = flat_u[i:i + step]
        r = (c + np.uint32(0x7FFF) + ((c >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
        flat_o[i:i + step] = r.astype(np.uint16)
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass
class Spec:
    """Shape and distribution of one synthetic decode batch."""
    name: str
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    q_dtype: str            # "f32" | "bf16"
    in_dtype: str           # dtype of appended k/v rows: "f32" | "bf16"
    kv_dtype: str           # cache dtype: "f32" | "bf16" | "e4m3" | "e5m2" | "int8"
    lengths: tuple          # ("uniform", lo, hi) | ("fixed", L) | ("lognormal", median, sigma, lo, hi) | ("list", (...))
    pool: tuple             # ("fixed", num_blocks) | ("double_unique", round_to)
    share_group: int = 0    # sequences per prefix-sharing group (0 = none)
    share_blocks: int = 0   # whole blocks of shared prefix per group
    max_blocks_per_seq: int | None = None   # table width; default ceil(max length / block size)
    seed: int = BASE_SEED


def config_spec(i: int) -> Spec:
    """The five standard workloads (0 tiny fp32, 1 Llama-3-8B bf16, 2 long bf16,
    3 mixed batch with shared prefixes bf16, 4 Qwen2.5-14B FP8-e4m3)."""
    if i == 0:
        return Spec("tiny_fp32", 4, 8, 2, 64, 16, "f32", "f32", "f32",
                    ("uniform", 1, 64), ("fixed", 32), max_blocks_per_seq=4, seed=BASE_SEED + 0)
    if i == 1:
        return Spec("llama3_8b_bf16", 64, 32, 8, 128, 16, "bf16", "bf16", "bf16",
                    ("uniform", 1024, 1280), ("fixed", 8192), max_blocks_per_seq=80, seed=BASE_SEED + 1)
    if i == 2:
        return Spec("long_16x8192_bf16", 16, 32, 8, 128, 16, "bf16", "bf16", "bf16",
                    ("fixed", 8192), ("fixed", 16384), max_blocks_per_seq=512, seed=BASE_SEED + 2)
    if i == 3:
        return Spec("mixed_prefix_bf16", 256, 32, 8, 128, 16, "bf16", "bf16", "bf16",
                    ("lognormal", 2300, 0.75, 100, 12000), ("double_unique", 1024),
                    share_group=8, share_blocks=64, max_blocks_per_seq=750, seed=BASE_SEED + 3)
    if i == 4:
        return Spec("qwen25_14b_fp8", 128, 40, 8, 128, 16, "bf16", "bf16", "e4m3",
                    ("uniform", 1024, 1280), ("fixed", 16384), max_blocks_per_seq=80, seed=BASE_SEED + 4)
    raise ValueError(f"unknown config {i}")


@dataclass
class DecodeBatch:
    spec: Spec
    num_blocks: int
    max_blocks_per_seq: int
    scale: np.float32
    k_scale: np.float32
    v_scale: np.float32
    seq_lens: np.ndarray          # int32 [S]
    block_tables: np.ndarray      # int32 [S, MB], -1 padded
    q: np.ndarray                 # [S, Hq, d]   float32 or uint16 (bf16 bits)
    hist_k: np.ndarray            # [T, Hkv, d]  float32 or uint16
    hist_v: np.ndarray
    hist_slots: np.ndarray        # int64 [T]
    new_k: np.ndarray             # [S, Hkv, d]
    new_v: np.ndarray
    new_slots: np.ndarray         # int64 [S]
    shared_blocks: int = 0        # physical blocks referenced by more than one sequence
    extra: dict = field(default_factory=dict)

    @property
    def num_seqs(self):
        return self.spec.num_seqs

    @property
    def group(self):
        return self.spec.num_heads // self.spec.num_kv_heads

    def nblocks(self) -> np.ndarray:
        bs = self.spec.block_size
        return (self.seq_lens.astype(np.int64) + bs - 1) // bs

    def unique_blocks(self) -> int:
        nb = self.nblocks()
        ids = np.concatenate([self.block_tables[s, :nb[s]] for s in range(self.num_seqs)]) if nb.sum() else np.zeros(0, np.int32)
        return int(np.unique(ids).size)


def _draw_lengths(spec: Spec, rng: np.random.Generator) -> np.ndarray:
    kind = spec.lengths[0]
    S = spec.num_seqs
    if kind == "uniform":
        lo, hi = spec.lengths[1], spec.lengths[2]
        return rng.integers(lo, hi + 1, size=S).astype(np.int32)
    if kind == "fixed":
        return np.full(S, spec.lengths[1], dtype=np.int32)
    if kind == "lognormal":
        median, sigma, lo, hi = spec.lengths[1:]
        x = rng.lognormal(mean=math.log(median), sigma=sigma, size=S)
        return np.clip(np.rint(x), lo, hi).astype(np.int32)
    if kind == "list":
        v = np.asarray(spec.lengths[1], dtype=np.int32)
        assert v.size == S
        return v.copy()
    raise ValueError(kind)


def _normal(rng, shape, dtype_name):
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if dtype_name == "bf16":
        return f32_to_bf16_bits(x)
    return x


def _absmax(x: np.ndarray, dtype_name: str) -> np.float32:
    if x.size == 0:
        return np.float32(0)
    if dtype_name == "bf16":
        # |bf16| ordering equals ordering of the magnitude bits
        m = int((x & np.uint16(0x7FFF)).max())
        return np.float32(bf16_bits_to_f32(np.array([m], dtype=np.uint16))[0])
    return np.float32(np.abs(x).max())


def _cache_scales(kv_dtype, in_dtype, hist_k, hist_v, new_k, new_v):
    """Per-tensor scales of an 8-bit cache: the absmax of every K (V) value written to the cache
    maps to the format's largest finite value (448 for E4M3, 57344 for E5M2, 127 for INT8);
    1 for f32 / bf16 caches."""
    if kv_dtype in ("e4m3", "e5m2", "int8"):
        top = np.float32({"e4m3": 448.0, "e5m2": 57344.0, "int8": 127.0}[kv_dtype])
        k_scale = np.float32(max(_absmax(hist_k, in_dtype), _absmax(new_k, in_dtype)) / top)
        v_scale = np.float32(max(_absmax(hist_v, in_dtype), _absmax(new_v, in_dtype)) / top)
        return k_scale, v_scale
    return np.float32(1.0), np.float32(1.0)


@dataclass
class Layout:
    """Lengths and block tables of a batch, before any tensor is drawn."""
    seq_lens: np.ndarray          # int32 [S]
    block_tables: np.ndarray      # int32 [S, MB], -1 padded
    num_blocks: int
    shared_n: np.ndarray          # int64 [S]: leading blocks taken from the group's shared prefix
    groups: list                  # [(members, blocks in the group's shared prefix)]


def _layout(spec: Spec, rng: np.random.Generator) -> Layout:
    S, bs = spec.num_seqs, spec.block_size
    seq_lens = _draw_lengths(spec, rng)
    nb = (seq_lens.astype(np.int64) + bs - 1) // bs
    MB = spec.max_blocks_per_seq or int(max(1, nb.max()))
    assert nb.max() <= MB, "table width too small for the drawn lengths"

    # Which logical blocks are shared: whole blocks strictly before the block
    # holding the new token (position L-1), at most share_blocks of them.
    shared_n = np.zeros(S, dtype=np.int64)
    if spec.share_group > 1:
        shared_n = np.minimum(spec.share_blocks, np.maximum(seq_lens.astype(np.int64) - 1, 0) // bs)
    groups = []
    if spec.share_group > 1:
        for g0 in range(0, S, spec.share_group):
            members = list(range(g0, min(S, g0 + spec.share_group)))
            groups.append((members, int(shared_n[members].max()) if members else 0))
    unique = sum(n for _, n in groups) + int((nb - shared_n).sum())

    if spec.pool[0] == "fixed":
        num_blocks = int(spec.pool[1])
    elif spec.pool[0] == "double_unique":
        r = int(spec.pool[1])
        num_blocks = int(-(-2 * unique // r) * r)
    else:
        raise ValueError(spec.pool)
    assert unique <= num_blocks, "pool too small"

    perm = rng.permutation(num_blocks).astype(np.int32)
    nxt = 0
    tables = np.full((S, MB), -1, dtype=np.int32)
    if groups:
        for members, gmax in groups:
            prefix = perm[nxt:nxt + gmax]
            nxt += gmax
            for s in members:
                n = int(shared_n[s])
                tables[s, :n] = prefix[:n]
                own = int(nb[s]) - n
                tables[s, n:n + own] = perm[nxt:nxt + own]
                nxt += own
    else:
        for s in range(S):
            n = int(nb[s])
            tables[s, :n] = perm[nxt:nxt + n]
            nxt += n
    assert nxt == unique
    return Layout(seq_lens, tables, num_blocks, shared_n, groups)


def batch_layout(spec: Spec, seed: int | None = None) -> Layout:
    """The lengths and tables ``build_batch`` draws for ``spec`` (same seed, same values)."""
    return _layout(spec, np.random.default_rng(spec.seed if seed is None else seed))


def build_batch(spec: Spec, seed: int | None = None) -> DecodeBatch:
    """Draw one batch. Draw order: lengths, pool permutation, q, K, V, new k, new v."""
    rng = np.random.default_rng(spec.seed if seed is None else seed)
    assert spec.num_heads % spec.num_kv_heads == 0
    lay = _layout(spec, rng)
    groups = lay.groups
    shared = int(sum(n for members, n in groups if len(members) > 1)) if groups else 0
    return _draw_tensors(spec, rng, lay.seq_lens, lay.block_tables, lay.num_blocks, shared)


def batch_from_tables(spec: Spec, block_tables: np.ndarray, seq_lens: np.ndarray, num_blocks: int,
                      seed: int | None = None) -> DecodeBatch:
    """A batch over given tables (e.g. a block manager's, with forks sharing blocks): q, the
    history rows of every slot of every referenced block and the new token rows are drawn as in
    ``build_batch`` (same order), the new token of sequence s at position seq_lens[s] - 1."""
    rng = np.random.default_rng(spec.seed if seed is None else seed)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    assert sl.shape == (spec.num_seqs,) and bt.shape[0] == spec.num_seqs
    nb = (sl.astype(np.int64) + spec.block_size - 1) // spec.block_size
    counts = {}
    for s in range(spec.num_seqs):
        for j in range(int(nb[s])):
            counts[int(bt[s, j])] = counts.get(int(bt[s, j]), 0) + 1
    shared = sum(1 for c in counts.values() if c > 1)
    return _draw_tensors(spec, rng, sl, bt, int(num_blocks), shared)


def _draw_tensors(spec: Spec, rng, seq_lens, tables, num_blocks, shared) -> DecodeBatch:
    S, Hq, Hkv, d, bs = spec.num_seqs, spec.num_heads, spec.num_kv_heads, spec.head_dim, spec.block_size
    MB = tables.shape[1]
    nb = (seq_lens.astype(np.int64) + bs - 1) // bs

    # referenced physical blocks in first-use order (shared ones once)
    ref = []
    seen = set()
    for s in range(S):
        for j in range(int(nb[s])):
            p = int(tables[s, j])
            if p not in seen:
                seen.add(p)
                ref.append(p)
    ref = np.asarray(ref, dtype=np.int64)
    hist_slots = (ref[:, None] * bs + np.arange(bs, dtype=np.int64)[None, :]).reshape(-1)

    q = _normal(rng, (S, Hq, d), spec.q_dtype)
    T = hist_slots.size
    hist_k = _normal(rng, (T, Hkv, d), spec.in_dtype)
    hist_v = _normal(rng, (T, Hkv, d), spec.in_dtype)
    new_k = _normal(rng, (S, Hkv, d), spec.in_dtype)
    new_v = _normal(rng, (S, Hkv, d), spec.in_dtype)

    new_slots = np.full(S, -1, dtype=np.int64)
    for s in range(S):
        L = int(seq_lens[s])
        if L > 0:
            pos = L - 1
            new_slots[s] = int(tables[s, pos // bs]) * bs + pos % bs

    k_scale, v_scale = _cache_scales(spec.kv_dtype, spec.in_dtype, hist_k, hist_v, new_k, new_v)
    scale = np.float32(1.0 / math.sqrt(d))
    return DecodeBatch(spec, num_blocks, MB, scale, k_scale, v_scale, seq_lens, tables, q,
                       hist_k, hist_v, hist_slots, new_k, new_v, new_slots, shared_blocks=shared)


def config_batch(i: int, **overrides) -> DecodeBatch:
    """Batch of standard workload ``i``; keyword overrides replace Spec fields
    (e.g. ``num_seqs=8`` for a cut-down copy with the same distributions)."""
    spec = config_spec(i)
    for k, v in overrides.items():
        setattr(spec, k, v)
    return build_batch(spec)


def subset_tokens(batch: DecodeBatch, seqs) -> np.ndarray:
    """Indices of history rows whose slots belong to blocks referenced by ``seqs``."""
    bs = batch.spec.block_size
    nb = batch.nblocks()
    blocks = set()
    for s in seqs:
        blocks.update(int(p) for p in batch.block_tables[s, :nb[s]])
    blk = batch.hist_slots // bs
    return np.nonzero(np.isin(blk, np.fromiter(blocks, dtype=np.int64, count=len(blocks))))[0]


def with_cache_dtype(batch: DecodeBatch, kv_dtype: str) -> DecodeBatch:
    """The same batch (lengths, tables, q, K, V, new rows: the arrays are shared, not copied) with
    another cache dtype and that dtype's per-tensor scales: what ``build_batch`` draws for the spec
    with ``kv_dtype`` replaced, without drawing the tensors again."""
    import copy
    sp = copy.copy(batch.spec)
    if kv_dtype != sp.kv_dtype:
        if sp.in_dtype != "bf16" or kv_dtype not in ("bf16", "e4m3", "e5m2", "int8"):
            raise ValueError(f"cannot re-type a {sp.in_dtype}-row batch to a {kv_dtype} cache")
        sp.kv_dtype = kv_dtype
        sp.name = f"{sp.name}_{kv_dtype}kv"
    b = copy.copy(batch)
    b.spec = sp
    b.k_scale, b.v_scale = _cache_scales(kv_dtype, sp.in_dtype, batch.hist_k, batch.hist_v, batch.new_k,
                                         batch.new_v)
    b.extra = dict(batch.extra)
    return b
