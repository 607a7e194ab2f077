"""Algorithmic byte counts of one decode step (host-side arithmetic only).

KV bytes per cached token = layers x kv_heads x head_dim x 2 (K and V) x
bytes per element: 32 x 8 x 128 x 2 x 2 = 131072 B = 128 KB for a 32-layer,
8-KV-head, head_dim 128 fp16/bf16 model, 4 KB per token per layer
("vLLM inference cost optimisation", developer.aliyun.com, section 2.1; the
wzjinhao.cn vLLM write-up, section 2.1, gives the same 4 KB per token per layer).
"""
from __future__ import annotations

import numpy as np

ELT = {"f32": 4, "bf16": 2, "e4m3": 1, "e5m2": 1, "int8": 1}


def kv_bytes_per_token(layers: int, kv_heads: int, head_dim: int, elt_bytes: int) -> int:
    return layers * kv_heads * head_dim * 2 * elt_bytes


def decode_bytes(seq_lens, block_tables, num_heads, num_kv_heads, head_dim, block_size, kv_dtype, q_dtype) -> dict:
    """Bytes paged attention must move for one call.

    kv_unique   every distinct physical block referenced, whole blocks, K and V
    kv_logical  sum over sequences of seq_len tokens of K and V (shared blocks counted per reader)
    q_out       q read plus out written
    tables      block-table entries read plus seq_lens
    total       kv_unique + q_out + tables (the roofline numerator)
    """
    sl = np.asarray(seq_lens, dtype=np.int64)
    bt = np.asarray(block_tables)
    nb = (sl + block_size - 1) // block_size
    per_tok = 2 * num_kv_heads * head_dim * ELT[kv_dtype]
    ids = np.concatenate([bt[s, :nb[s]] for s in range(sl.size)]) if nb.sum() else np.zeros(0, np.int64)
    unique_blocks = int(np.unique(ids).size)
    kv_unique = unique_blocks * block_size * per_tok
    kv_logical = int(sl.sum()) * per_tok
    q_out = 2 * sl.size * num_heads * head_dim * ELT[q_dtype]
    tables = int(nb.sum()) * 4 + 4 * sl.size
    return dict(kv_unique=kv_unique, kv_logical=kv_logical, q_out=q_out, tables=tables,
                unique_blocks=unique_blocks, total=kv_unique + q_out + tables)


def plan_bytes(seq_lens, block_size, plan) -> dict:
    """Change in the bytes a shared-prefix decode reads besides K/V, q and out: the block-table
    entries of the shared blocks are not read (their group's row is, once per group), and the
    plan's arrays are (members, offsets, row lengths, per-sequence shared counts). Returns
    {"tables_saved": bytes, "plan": bytes}."""
    shared = np.asarray(plan.shared, dtype=np.int64)
    groups = int(plan.num_groups)
    members = int(np.asarray(plan.offsets)[groups]) if groups else 0
    group_blocks = int((np.asarray(plan.lens[:groups], dtype=np.int64) // block_size).sum()) if groups else 0
    return {"tables_saved": 4 * int(shared.sum()),
            "plan": 4 * (group_blocks + members + (groups + 1) + groups + shared.size)}


def append_bytes(num_tokens, num_kv_heads, head_dim, in_dtype, kv_dtype) -> int:
    """reshape_and_cache: read the K and V rows and their slot, write the cache rows."""
    rows = 2 * num_tokens * num_kv_heads * head_dim
    return rows * ELT[in_dtype] + rows * ELT[kv_dtype] + 8 * num_tokens


def decode_flops(seq_lens, num_heads, head_dim) -> int:
    """q.K and p.V multiply-adds, 2 flops each: 4 * heads * head_dim per cached token."""
    return 4 * int(np.asarray(seq_lens, dtype=np.int64).sum()) * num_heads * head_dim
