"""Turn a workload description into the host arrays the kernels consume.

Runs the block allocator step by step the way a serving engine would for one
iteration: sequences that already hold their earlier context, the new tokens
of this step appended one by one (taking blocks on demand and copying shared
blocks before they are written), then one attention call over everything.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .allocator import BlockAllocator


@dataclass
class Batch:
    block_tables: np.ndarray       # int32 [S, max_blocks]
    context_lens: np.ndarray       # int32 [S], includes this step's tokens
    query_start_loc: np.ndarray | None  # int32 [S+1], None = one query token per sequence
    slot_mapping: np.ndarray       # int64 [T_new] slots of this step's new tokens
    cow_pairs: np.ndarray          # int64 [P, 2] (src, dst) block copies before the writes
    max_query_len: int
    allocator: BlockAllocator

    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0


def build_batch(wl) -> Batch:
    """``wl`` is a ``workloads.Workload``."""
    alloc = BlockAllocator(wl.num_blocks, wl.block_size, wl.free_order)
    slots: list[int] = []
    cows: list[tuple[int, int]] = []
    sids: list[int] = []

    def append(sid):
        s, cow = alloc.append_slot(sid)
        slots.append(s)
        if cow is not None:
            cows.append(cow)

    if wl.kind in ("decode", "mixed"):
        for L, Q in zip(wl.context_lens, wl.query_lens):
            if L < Q:  # empty context: the query token has no K/V to write (padding slot)
                sid = alloc.new_sequence(L)
                slots.extend([-1] * Q)
            else:
                sid = alloc.new_sequence(L - Q)
                for _ in range(Q):
                    append(sid)
            sids.append(sid)
        qlens = list(wl.query_lens)
    elif wl.kind == "shared_prefix":
        for p in range(wl.num_prompts):
            root = alloc.new_sequence(wl.prompt_len)
            group = [root] + [alloc.fork(root) for _ in range(wl.samples - 1)]
            sids.extend(group)
        for sid, tail in zip(sids, wl.tails):
            for _ in range(tail):
                append(sid)
        qlens = [1] * len(sids)
    else:
        raise ValueError(wl.kind)

    qsl = None
    if any(q != 1 for q in qlens):
        qsl = np.zeros(len(qlens) + 1, dtype=np.int32)
        qsl[1:] = np.cumsum(qlens)
    return Batch(
        block_tables=alloc.block_tables_array(sids),
        context_lens=alloc.context_lens_array(sids),
        query_start_loc=qsl,
        slot_mapping=np.asarray(slots, dtype=np.int64),
        cow_pairs=np.asarray(cows, dtype=np.int64).reshape(-1, 2),
        max_query_len=max(qlens) if qlens else 0,
        allocator=alloc,
    )


def shared_prefix_groups(block_tables: np.ndarray, context_lens: np.ndarray, block_size: int,
                         min_shared_blocks: int = 1):
    """Group consecutive sequences whose block tables start with the same
    physical blocks (forks of one prompt share them until they diverge).

    Returns ``(group_start, group_shared_blocks)``, int32 arrays of G+1 and G
    entries covering every sequence: group j is sequences
    group_start[j] .. group_start[j+1]-1, which share their first
    group_shared_blocks[j] block-table entries.  Only blocks that every member
    has filled count (shared blocks * block_size <= each member's context).
    A sequence that shares fewer than ``min_shared_blocks`` blocks with the
    sequence before it starts a new group; groups of one sequence get 0.
    """
    bt = np.asarray(block_tables)
    lens = np.asarray(context_lens, dtype=np.int64)
    n = lens.shape[0]
    starts, shared = [0], []
    s = 0
    while s < n:
        p = int(lens[s] // block_size)
        e = s + 1
        while e < n:
            lim = min(p, int(lens[e] // block_size))
            same = bt[s, :lim] == bt[e, :lim]
            c = lim if same.all() else int(np.argmin(same))
            if c < min_shared_blocks:
                break
            p = c
            e += 1
        shared.append(p if e - s > 1 else 0)
        starts.append(e)
        s = e
    return np.asarray(starts, dtype=np.int32), np.asarray(shared, dtype=np.int32)


def staged_blocks_needed(query_start_loc, context_lens, block_size) -> int:
    """Blocks pa_decode_fp8_rows stages for a batch over an FP8 cache: those of
    the sequences with more than one query row (host arrays or CPU tensors)."""
    qsl = np.asarray(query_start_loc, dtype=np.int64)
    cl = np.asarray(context_lens, dtype=np.int64)
    q = qsl[1:] - qsl[:-1]
    return int(((cl + block_size - 1) // block_size)[(q > 1) & (cl > 0)].sum())
