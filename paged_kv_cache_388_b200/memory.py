"""KV-cache memory accounting: paged blocks versus contiguous reservation.

The pages' argument for paging is memory: reserving a contiguous region of the
maximum length per request wastes most of it, while blocks waste at most the
unused tail of each sequence's last block ("核心概念", sections 传统方法的痛点 and
PagedAttention 的优势总结; "理解 vLLM PagedAttention", section 四).  These helpers
measure both on a set of context lengths, counting token slots.
"""
from __future__ import annotations

import numpy as np


def paged_usage(lengths, block_size: int) -> dict:
    """Slots held when each sequence takes ceil(L / block_size) private blocks."""
    L = np.asarray(lengths, dtype=np.int64)
    slots = int((-(-L // block_size) * block_size).sum())
    tokens = int(L.sum())
    return {"tokens": tokens, "slots": slots, "waste_frac": (slots - tokens) / slots if slots else 0.0,
            "utilization": tokens / slots if slots else 1.0}


def reserved_usage(lengths, max_len: int) -> dict:
    """Slots held when each sequence reserves max_len contiguous slots up front."""
    L = np.asarray(lengths, dtype=np.int64)
    if (L > max_len).any():
        raise ValueError("a length exceeds the reservation")
    slots = int(L.size) * int(max_len)
    tokens = int(L.sum())
    return {"tokens": tokens, "slots": slots, "waste_frac": (slots - tokens) / slots if slots else 0.0,
            "utilization": tokens / slots if slots else 1.0}


def pool_usage(allocator) -> dict:
    """Live pool of a BlockAllocator: physical slots in use (shared blocks once)
    against the tokens its sequences hold (shared prefixes counted per sequence)."""
    u = allocator.usage()
    slots, tokens = u["slots_in_use"], u["tokens_logical"]
    return {"tokens_logical": tokens, "slots": slots, "blocks": u["blocks_in_use"],
            "logical_per_slot": tokens / slots if slots else 0.0}


def waste_report(lengths, block_size: int, max_len: int) -> dict:
    p = paged_usage(lengths, block_size)
    r = reserved_usage(lengths, max_len)
    return {"paged": p, "reserved": r, "slot_ratio": r["slots"] / p["slots"] if p["slots"] else 0.0}
