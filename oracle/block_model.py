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


def prefix_plan(tables, lens, bs: int, max_group: int):
    """Shared-prefix groups of one decode batch: [(members, group_table, shared)], where
    ``shared[i]`` = leading blocks member i reads through ``group_table`` instead of its own.

    Reading of the pages' block-granular prefix sharing (wzjinhao.cn write-up, section 2.3;
    "vLLM inference cost optimisation", section 11): sequences whose tables hold the same
    physical block hold the same tokens there, so one pass over that block can serve all of
    them. Only full blocks count (j + 1 <= len / bs). Candidates: sequences whose first block
    is full, bucketed by its id (buckets in order of first appearance), each bucket cut into
    chunks of max_group in index order; a chunk of one is left alone. Within a chunk, walk
    j = 0, 1, ...: among the members still sharing, take the id held at j by the most of
    them (ties: the first such member's id); stop when no id is held by two; the members
    holding it stay. No arithmetic of the attention lives here."""
    def full(s, j):
        return j < len(tables[s]) and (j + 1) * bs <= lens[s] and tables[s][j] >= 0

    buckets, order = {}, []
    for s in range(len(lens)):
        if full(s, 0):
            b = int(tables[s][0])
            if b not in buckets:
                buckets[b] = []
                order.append(b)
            buckets[b].append(s)
    groups = []
    for b in order:
        members = buckets[b]
        for c0 in range(0, len(members), max(1, max_group)):
            chunk = members[c0:c0 + max(1, max_group)]
            if len(chunk) < 2:
                continue
            active, shared, table, j = list(chunk), {s: 0 for s in chunk}, [], 0
            while True:
                ids = [int(tables[s][j]) for s in active if full(s, j)]
                best, best_n = None, 1
                for x in ids:
                    if ids.count(x) > best_n:
                        best, best_n = x, ids.count(x)
                if best is None:
                    break
                table.append(best)
                active = [s for s in active if full(s, j) and tables[s][j] == best]
                for s in active:
                    shared[s] = j + 1
                j += 1
            groups.append((chunk, table, [shared[s] for s in chunk]))
    return groups
