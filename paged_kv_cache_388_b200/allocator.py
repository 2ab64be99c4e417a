"""Host-side block allocator: a free list of physical blocks plus refcounts.

This is the bookkeeping half of PagedAttention.  The KV cache of every
sequence is split into fixed-size blocks that live anywhere in one global pool
("核心概念", section 核心概念：块（Block）); each sequence keeps a block table that
maps its logical blocks to physical ones (section 逻辑视图与物理视图分离).  A block
is taken from the pool only when the last one is full (section 按需分配), so at
most one block per sequence is partly empty ("理解 vLLM PagedAttention", section
四).  Forked sequences share physical blocks through a reference count, and a
shared block is copied before it is written (section 六: copy-on-write).

The allocator runs on the host, off the timed path, and produces the inputs of
the device kernels: block tables, context lengths, slot mappings for
``pa_reshape_and_cache`` and (src, dst) pairs for ``pa_copy_blocks``.
"""
from __future__ import annotations

from collections import deque

import numpy as np


class PoolExhausted(RuntimeError):
    """No free physical block is left (the point where a serving engine would
    preempt a request)."""


class BlockAllocator:
    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        order = range(self.num_blocks) if free_order is None else free_order
        self._free = deque(int(b) for b in order)
        if len(self._free) != self.num_blocks or len(set(self._free)) != self.num_blocks:
            raise ValueError("free_order must be a permutation of range(num_blocks)")
        self._ref = np.zeros(self.num_blocks, dtype=np.int64)
        self._tables: dict[int, list[int]] = {}
        self._lens: dict[int, int] = {}
        self._next_id = 0

    # ---- pool state -------------------------------------------------------
    @property
    def num_free(self) -> int:
        return len(self._free)

    def refcount(self, block: int) -> int:
        return int(self._ref[block])

    def _take(self) -> int:
        if not self._free:
            raise PoolExhausted(f"all {self.num_blocks} blocks are in use")
        b = self._free.popleft()
        assert self._ref[b] == 0
        self._ref[b] = 1
        return b

    def _release(self, b: int) -> None:
        self._ref[b] -= 1
        assert self._ref[b] >= 0
        if self._ref[b] == 0:
            self._free.append(b)

    # ---- sequences ----------------------------------------------------------
    def new_sequence(self, num_tokens: int = 0) -> int:
        """Start a sequence whose first ``num_tokens`` tokens already have K/V
        (a prompt); takes ceil(num_tokens / bs) blocks."""
        nblk = -(-int(num_tokens) // self.block_size)
        if nblk > self.num_free:
            raise PoolExhausted(f"need {nblk} blocks, {self.num_free} free")
        sid = self._next_id
        self._next_id += 1
        self._tables[sid] = [self._take() for _ in range(nblk)]
        self._lens[sid] = int(num_tokens)
        return sid

    def fork(self, sid: int) -> int:
        """A new sequence sharing every block of ``sid`` (parallel sampling,
        beam search)."""
        child = self._next_id
        self._next_id += 1
        self._tables[child] = list(self._tables[sid])
        self._lens[child] = self._lens[sid]
        for b in self._tables[child]:
            self._ref[b] += 1
        return child

    def append_slot(self, sid: int):
        """Reserve the slot of the sequence's next token.

        Returns ``(slot, cow)``: ``cow`` is ``None`` or a ``(src, dst)`` pair
        that must be copied with ``pa_copy_blocks`` before the token's K/V are
        written, because the last block was shared.
        """
        bs = self.block_size
        table = self._tables[sid]
        pos = self._lens[sid]
        cow = None
        if pos % bs == 0:
            table.append(self._take())
        else:
            last = table[-1]
            if self._ref[last] > 1:
                fresh = self._take()
                self._ref[last] -= 1
                table[-1] = fresh
                cow = (last, fresh)
        self._lens[sid] = pos + 1
        return table[pos // bs] * bs + pos % bs, cow

    def free(self, sid: int) -> None:
        for b in self._tables.pop(sid):
            self._release(b)
        del self._lens[sid]

    def block_table(self, sid: int) -> list[int]:
        return list(self._tables[sid])

    def context_len(self, sid: int) -> int:
        return self._lens[sid]

    def sequences(self) -> list[int]:
        return list(self._tables)

    # ---- device inputs ------------------------------------------------------
    def block_tables_array(self, sids, max_blocks: int | None = None) -> np.ndarray:
        """int32 [len(sids), max_blocks]; entries past a sequence's last block
        are 0 and never read by the kernels."""
        rows = [self._tables[s] for s in sids]
        width = max((len(r) for r in rows), default=0) if max_blocks is None else max_blocks
        width = max(width, 1)
        out = np.zeros((len(rows), width), dtype=np.int32)
        for i, r in enumerate(rows):
            if len(r) > width:
                raise ValueError("max_blocks smaller than a block table")
            out[i, :len(r)] = r
        return out

    def context_lens_array(self, sids) -> np.ndarray:
        return np.asarray([self._lens[s] for s in sids], dtype=np.int32)

    # ---- memory accounting --------------------------------------------------
    def usage(self) -> dict:
        """Slots held vs tokens stored, counting each physical block once."""
        held = int(np.count_nonzero(self._ref))
        tokens_logical = sum(self._lens.values())
        return {
            "blocks_in_use": held,
            "slots_in_use": held * self.block_size,
            "tokens_logical": tokens_logical,
            "free_blocks": self.num_free,
        }
