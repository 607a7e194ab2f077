"""ctypes binding of the host block manager (include/pkv_blocks.h): argument marshalling only."""
from __future__ import annotations

import ctypes

import numpy as np

from . import PkvError, load_library

NO_BLOCKS, UNKNOWN_SEQ, DUPLICATE_SEQ, TABLE_FULL, HOST_ALLOC = 20, 21, 22, 23, 24

_bound = False


def _lib():
    global _bound
    lib = load_library()
    if not _bound:
        P, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        lib.pkv_bm_create.argtypes = [i32, i32, i32]
        lib.pkv_bm_create.restype = P
        lib.pkv_bm_destroy.argtypes = [P]
        lib.pkv_bm_destroy.restype = None
        lib.pkv_bm_add.argtypes = [P, i64, i32]
        lib.pkv_bm_fork.argtypes = [P, i64, i64]
        lib.pkv_bm_append.argtypes = [P, i64, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int32),
                                      ctypes.POINTER(ctypes.c_int32)]
        lib.pkv_bm_free.argtypes = [P, i64]
        lib.pkv_bm_num_free.argtypes = [P]
        lib.pkv_bm_seq_len.argtypes = [P, i64]
        lib.pkv_bm_ref_count.argtypes = [P, i32]
        lib.pkv_bm_step.argtypes = [P, P, i32, P, P, P, P, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
        lib.pkv_bm_tables.argtypes = [P, P, i32, P, P]
        lib.pkv_prefix_plan.argtypes = [P, P, i32, i32, i32, i32, P, P, P, P, P, ctypes.POINTER(ctypes.c_int)]
        lib.pkv_prefix_pass_inputs.argtypes = [P, P, i32, i32, i32, P, P, i32, P, i32, P, P, P, P]
        for n in ("pkv_bm_add", "pkv_bm_fork", "pkv_bm_append", "pkv_bm_free", "pkv_bm_num_free", "pkv_bm_seq_len",
                  "pkv_bm_ref_count", "pkv_bm_step", "pkv_bm_tables", "pkv_prefix_plan", "pkv_prefix_pass_inputs"):
            getattr(lib, n).restype = i32
        _bound = True
    return lib


class BlockManager:
    """Pool of `num_blocks` blocks of `block_size` tokens; tables `max_blocks_per_seq` wide.

    Status-returning calls return the C status (0 = ok, NO_BLOCKS, UNKNOWN_SEQ, ...)."""

    def __init__(self, num_blocks: int, block_size: int, max_blocks_per_seq: int):
        self._lib = _lib()
        self.block_size = block_size
        self.max_blocks = max_blocks_per_seq
        self._h = self._lib.pkv_bm_create(num_blocks, block_size, max_blocks_per_seq)
        if not self._h:
            raise PkvError("pkv_bm_create", 2)

    def close(self):
        if self._h:
            self._lib.pkv_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def add(self, seq_id: int, prompt_len: int) -> int:
        return self._lib.pkv_bm_add(self._h, seq_id, prompt_len)

    def fork(self, parent: int, child: int) -> int:
        return self._lib.pkv_bm_fork(self._h, parent, child)

    def append(self, seq_id: int):
        """(status, slot, cow_src, cow_dst)"""
        slot, src, dst = ctypes.c_int64(-1), ctypes.c_int32(-1), ctypes.c_int32(-1)
        st = self._lib.pkv_bm_append(self._h, seq_id, ctypes.byref(slot), ctypes.byref(src), ctypes.byref(dst))
        return st, slot.value, src.value, dst.value

    def free(self, seq_id: int) -> int:
        return self._lib.pkv_bm_free(self._h, seq_id)

    def num_free(self) -> int:
        return self._lib.pkv_bm_num_free(self._h)

    def seq_len(self, seq_id: int) -> int:
        return self._lib.pkv_bm_seq_len(self._h, seq_id)

    def ref_count(self, block: int) -> int:
        return self._lib.pkv_bm_ref_count(self._h, block)

    def step(self, seq_ids):
        """Append one token to each sequence; returns
        (status, slot_mapping int64[n], block_tables int32[n, max_blocks], seq_lens int32[n],
        cow_pairs int32[k, 2], n_done)."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = ids.size
        slots = np.full(n, -1, dtype=np.int64)
        tables = np.full((n, self.max_blocks), -1, dtype=np.int32)
        lens = np.zeros(n, dtype=np.int32)
        cows = np.full((max(n, 1), 2), -1, dtype=np.int32)
        n_cow, n_done = ctypes.c_int(0), ctypes.c_int(0)
        st = self._lib.pkv_bm_step(self._h, ids.ctypes.data, n, slots.ctypes.data, tables.ctypes.data,
                                   lens.ctypes.data, cows.ctypes.data, ctypes.byref(n_cow), ctypes.byref(n_done))
        return st, slots, tables, lens, cows[:n_cow.value].copy(), n_done.value

    def tables(self, seq_ids):
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        tables = np.full((ids.size, self.max_blocks), -1, dtype=np.int32)
        lens = np.zeros(ids.size, dtype=np.int32)
        st = self._lib.pkv_bm_tables(self._h, ids.ctypes.data, ids.size, tables.ctypes.data, lens.ctypes.data)
        return st, tables, lens


class PrefixPlan:
    """Output of pkv_prefix_plan: ``members[offsets[g]:offsets[g + 1]]`` share row g of
    ``tables`` (``lens[g]`` tokens); sequence s reads its first ``shared[s]`` blocks there."""

    def __init__(self, members, offsets, tables, lens, shared, num_groups):
        self.num_groups = num_groups
        self.members, self.offsets = members, offsets[: num_groups + 1]
        self.tables, self.lens, self.shared = tables[:num_groups], lens[:num_groups], shared

    def groups(self):
        """[(members, shared block ids, per-member shared counts)] in group order."""
        out = []
        for g in range(self.num_groups):
            m = self.members[self.offsets[g]:self.offsets[g + 1]].tolist()
            t = self.tables[g][self.tables[g] >= 0].tolist()
            out.append((m, t, [int(self.shared[s]) for s in m]))
        return out


def prefix_plan(block_tables, seq_lens, block_size: int, max_group: int) -> PrefixPlan:
    """Group the sequences of one decode batch by the full physical blocks they share
    (host arrays: block_tables int32 [n, max_blocks], seq_lens int32 [n])."""
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    n, mb = bt.shape
    members = np.zeros(n, dtype=np.int32)
    offsets = np.zeros(n + 1, dtype=np.int32)
    tables = np.full((max(n, 1), mb), -1, dtype=np.int32)
    lens = np.zeros(max(n, 1), dtype=np.int32)
    shared = np.zeros(n, dtype=np.int32)
    ng = ctypes.c_int(0)
    st = _lib().pkv_prefix_plan(bt.ctypes.data, sl.ctypes.data, n, mb, block_size, max_group, members.ctypes.data,
                                offsets.ctypes.data, tables.ctypes.data, lens.ctypes.data, shared.ctypes.data,
                                ctypes.byref(ng))
    if st != 0:
        raise PkvError("pkv_prefix_plan", st)
    return PrefixPlan(members, offsets, tables, lens, shared, ng.value)


def prefix_pass_inputs(block_tables, seq_lens, block_size: int, plan: PrefixPlan, query_heads_per_kv_head: int):
    """(col_seq int32 [groups, 8], col_limit int32 [groups, 8], suffix_tables, suffix_lens) for the
    two passes of a shared-prefix decode (pkv_prefix_pass_inputs)."""
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    n, mb = bt.shape
    g = plan.num_groups
    col_seq = np.full((max(g, 1), 8), -1, dtype=np.int32)
    col_limit = np.zeros((max(g, 1), 8), dtype=np.int32)
    suf_t = np.full((n, mb), -1, dtype=np.int32)
    suf_l = np.zeros(n, dtype=np.int32)
    members = np.ascontiguousarray(plan.members, dtype=np.int32)
    offsets = np.ascontiguousarray(plan.offsets, dtype=np.int32)
    shared = np.ascontiguousarray(plan.shared, dtype=np.int32)
    st = _lib().pkv_prefix_pass_inputs(bt.ctypes.data, sl.ctypes.data, n, mb, block_size, members.ctypes.data,
                                       offsets.ctypes.data, g, shared.ctypes.data, query_heads_per_kv_head,
                                       col_seq.ctypes.data, col_limit.ctypes.data, suf_t.ctypes.data,
                                       suf_l.ctypes.data)
    if st != 0:
        raise PkvError("pkv_prefix_pass_inputs", st)
    return col_seq[:g], col_limit[:g], suf_t, suf_l
