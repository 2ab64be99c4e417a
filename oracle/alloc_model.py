"""Block-allocation rules written as plain definitions -- test infrastructure.

The host allocator of the product builds block tables, slot mappings and
copy-on-write pairs; this model states the same rules in the most direct form
so the two can be compared entry by entry.

* A sequence of n tokens occupies ceil(n / bs) blocks; the waste is confined to
  the last block ("理解 vLLM PagedAttention", section 四: 100 tokens at block
  size 16 take 7 blocks, only the last partly used).
* Blocks are taken from the global pool only when needed: appending token p
  takes a new block exactly when p % bs == 0 ("核心概念", section 按需分配).
* Token p of a sequence with table T is stored at slot T[p // bs] * bs + p % bs
  ("核心概念", section 逻辑视图与物理视图分离).
* Forked sequences point at the same physical blocks, counted by a reference
  count; a shared block is copied before it is written ("理解 vLLM
  PagedAttention", section 六; "PagedAttention 实战", section PagedAttention 的核心,
  item 3 块级共享).
"""
from __future__ import annotations


def blocks_needed(n: int, bs: int) -> int:
    return (n + bs - 1) // bs


def slot_of(table, pos: int, bs: int) -> int:
    return table[pos // bs] * bs + pos % bs


class PoolModel:
    """Free list popped from the front, refcount per physical block."""

    def __init__(self, free_order, bs: int):
        self.free = [int(b) for b in free_order]
        self.bs = bs
        self.ref = {}
        self.tables = {}
        self.lens = {}
        self.copies = []

    def _take(self) -> int:
        b = self.free.pop(0)
        self.ref[b] = 1
        return b

    def new_sequence(self, sid, n: int):
        self.tables[sid] = [self._take() for _ in range(blocks_needed(n, self.bs))]
        self.lens[sid] = n

    def fork(self, parent, child):
        self.tables[child] = list(self.tables[parent])
        self.lens[child] = self.lens[parent]
        for b in self.tables[child]:
            self.ref[b] += 1

    def append(self, sid) -> int:
        p = self.lens[sid]
        table = self.tables[sid]
        if p % self.bs == 0:
            table.append(self._take())
        else:
            last = table[-1]
            if self.ref[last] > 1:
                fresh = self._take()
                self.copies.append((last, fresh))
                self.ref[last] -= 1
                table[-1] = fresh
        self.lens[sid] = p + 1
        return slot_of(table, p, self.bs)
