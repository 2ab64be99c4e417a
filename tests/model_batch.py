"""Oracle-side construction of a workload's batch from the plain allocation
rules in oracle/alloc_model.py (never from the product allocator)."""
import numpy as np

from oracle.alloc_model import PoolModel


def model_batch(wl):
    m = PoolModel(wl.free_order, wl.block_size)
    slots, sids = [], []
    if wl.kind in ("decode", "mixed"):
        for i, (L, Q) in enumerate(zip(wl.context_lens, wl.query_lens)):
            if L < Q:
                m.new_sequence(i, L)
                slots.extend([-1] * Q)
            else:
                m.new_sequence(i, L - Q)
                for _ in range(Q):
                    slots.append(m.append(i))
            sids.append(i)
        qlens = list(wl.query_lens)
    else:
        for p in range(wl.num_prompts):
            root = (p, 0)
            m.new_sequence(root, wl.prompt_len)
            sids.append(root)
            for s in range(1, wl.samples):
                m.fork(root, (p, s))
                sids.append((p, s))
        for sid, tail in zip(sids, wl.tails):
            for _ in range(tail):
                slots.append(m.append(sid))
        qlens = [1] * len(sids)
    width = max(len(m.tables[s]) for s in sids)
    bt = np.zeros((len(sids), width), np.int32)
    for i, s in enumerate(sids):
        bt[i, : len(m.tables[s])] = m.tables[s]
    cl = np.asarray([m.lens[s] for s in sids], np.int32)
    qsl = None
    if any(q != 1 for q in qlens):
        qsl = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    return dict(block_tables=bt, context_lens=cl, query_start_loc=qsl,
                slot_mapping=np.asarray(slots, np.int64),
                cow_pairs=np.asarray(m.copies, np.int64).reshape(-1, 2))
