"""Plain model of the paged KV cache's block pool (test infrastructure: only tests/ use it).

It restates, in the simplest Python, what the host block manager must do. The pages
("vLLM inference cost optimisation", developer.aliyun.com, sections 4 and 4.1;
wzjinhao.cn vLLM write-up, sections 2.1 and 2.3) fix the data: a pool of fixed-size
blocks, a per-sequence table from logical block i to a physical block, a new block only
when the last one is full, and whole blocks shared between sequences with a common
prefix. They give no allocator; the policy read here (and documented with the C ABI):

* free list: FIFO, initially 0..num_blocks-1; take from the front, return to the back;
* fork: the child copies the parent's table, each block's count +1;
* append at position L: L % bs == 0 -> a fresh block; otherwise, if the last block is
  shared (count > 1), copy on write: a fresh block replaces it in this table, the old
  count -1, the pair (old, fresh) is reported; slot = table[-1] * bs + L % bs;
* free: counts -1, blocks reaching 0 return to the free list in table order.

No arithmetic of the attention lives here.
"""
from __future__ import annotations

from collections import deque

OK, NO_BLOCKS, UNKNOWN_SEQ, DUPLICATE_SEQ, TABLE_FULL = 0, 20, 21, 22, 23


class BlockModel:
    def __init__(self, num_blocks: int, block_size: int, max_blocks_per_seq: int):
        self.num_blocks = num_blocks
        self.bs = block_size
        self.max_blocks = max_blocks_per_seq
        self.free = deque(range(num_blocks))
        self.refs = [0] * num_blocks
        self.seqs = {}   # id -> [length, table]

    def _take(self) -> int:
        b = self.free.popleft()
        self.refs[b] = 1
        return b

    def add(self, sid: int, prompt_len: int) -> int:
        if sid in self.seqs:
            return DUPLICATE_SEQ
        need = -(-prompt_len // self.bs)
        if need > self.max_blocks:
            return TABLE_FULL
        if need > len(self.free):
            return NO_BLOCKS
        self.seqs[sid] = [prompt_len, [self._take() for _ in range(need)]]
        return OK

    def fork(self, parent: int, child: int) -> int:
        if parent not in self.seqs:
            return UNKNOWN_SEQ
        if child in self.seqs:
            return DUPLICATE_SEQ
        length, table = self.seqs[parent]
        for b in table:
            self.refs[b] += 1
        self.seqs[child] = [length, list(table)]
        return OK

    def append(self, sid: int):
        """(status, slot, cow_src, cow_dst)"""
        if sid not in self.seqs:
            return UNKNOWN_SEQ, -1, -1, -1
        length, table = self.seqs[sid]
        off = length % self.bs
        src = dst = -1
        if off == 0:
            if len(table) >= self.max_blocks:
                return TABLE_FULL, -1, -1, -1
            if not self.free:
                return NO_BLOCKS, -1, -1, -1
            table.append(self._take())
        elif self.refs[table[-1]] > 1:
            if not self.free:
                return NO_BLOCKS, -1, -1, -1
            src, dst = table[-1], self._take()
            self.refs[src] -= 1
            table[-1] = dst
        self.seqs[sid][0] = length + 1
        return OK, table[-1] * self.bs + off, src, dst

    def free_seq(self, sid: int) -> int:
        if sid not in self.seqs:
            return UNKNOWN_SEQ
        for b in self.seqs.pop(sid)[1]:
            self.refs[b] -= 1
            if self.refs[b] == 0:
                self.free.append(b)
        return OK

    def step(self, ids):
        """(status, slots, tables, lens, cow_pairs, n_done): append to each, in order."""
        slots, cows = [], []
        for i, sid in enumerate(ids):
            st, slot, src, dst = self.append(sid)
            if st != OK:
                return st, slots, None, None, cows, i
            slots.append(slot)
            if src >= 0:
                cows.append((src, dst))
        tables = [self.seqs[s][1] + [-1] * (self.max_blocks - len(self.seqs[s][1])) for s in ids]
        return OK, slots, tables, [self.seqs[s][0] for s in ids], cows, len(ids)
