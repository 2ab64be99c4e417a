"""Host block allocator (product) against the pages' worked examples and the
oracle's plain allocation rules (bit-exact tables, slots and CoW pairs)."""
import numpy as np
import pytest

import workloads
from model_batch import model_batch
from oracle_pins import golden
from paged_kv_cache_388_b200.allocator import BlockAllocator, PoolExhausted
from paged_kv_cache_388_b200.batch import build_batch


def test_worked_block_table_and_growth():
    g = golden("on_demand_growth.json")
    a = BlockAllocator(20, g["block_size"], g["free_order_head"] + list(range(10, 20))
                       + [0, 3, 4, 6, 7, 9])
    sid = a.new_sequence(0)
    for n in range(1, 65):
        slot, cow = a.append_slot(sid)
        assert cow is None
        if str(n) in g["table_after_tokens"]:
            assert a.block_table(sid) == g["table_after_tokens"][str(n)]
    w = golden("block_table_worked_example.json")
    assert a.block_table(sid) == w["block_table"]
    # replay: slots of tokens 0..63 match the hand-derived ones
    b = BlockAllocator(20, 16, g["free_order_head"] + list(range(10, 20)) + [0, 3, 4, 6, 7, 9])
    s2 = b.new_sequence(0)
    slots = [b.append_slot(s2)[0] for _ in range(64)]
    for tok, slot in w["slots_derived_by_hand"].items():
        assert slots[int(tok)] == slot


def test_block_count_example():
    g = golden("block_count_worked_example.json")
    a = BlockAllocator(16, g["block_size"])
    sid = a.new_sequence(g["tokens"])
    assert len(a.block_table(sid)) == g["blocks"]
    u = a.usage()
    assert u["slots_in_use"] - g["tokens"] < g["block_size"]


@pytest.mark.parametrize("cfg", workloads.SMALL_CONFIGS + ("3", "4", "4cow", "5", "5bs32"))
def test_batch_matches_oracle_rules(cfg):
    wl = workloads.make(cfg)
    b = build_batch(wl)
    m = model_batch(wl)
    assert np.array_equal(b.block_tables, m["block_tables"])
    assert np.array_equal(b.context_lens, m["context_lens"])
    assert np.array_equal(b.slot_mapping, m["slot_mapping"])
    assert np.array_equal(b.cow_pairs, m["cow_pairs"])
    if m["query_start_loc"] is None:
        assert b.query_start_loc is None
    else:
        assert np.array_equal(b.query_start_loc, m["query_start_loc"])
    # slots unique (several writers to one slot would make the result ambiguous)
    real = b.slot_mapping[b.slot_mapping >= 0]
    assert len(set(real.tolist())) == real.size
    # refcounts: each block in use is referenced by exactly refcount tables
    refs = np.zeros(wl.num_blocks, np.int64)
    for i, L in enumerate(b.context_lens):
        nblk = -(-int(L) // wl.block_size)
        for pb in b.block_tables[i, :nblk]:
            refs[pb] += 1
    for pb in range(wl.num_blocks):
        assert refs[pb] == b.allocator.refcount(pb)
    assert b.allocator.num_free + np.count_nonzero(refs) == wl.num_blocks


def test_empty_context_gets_padding_slot():
    wl = workloads.decode_workload("edge", 1, [0, 1, 16, 17], 8, 2, 64, 16, "f32")
    b = build_batch(wl)
    m = model_batch(wl)
    assert b.slot_mapping[0] == -1 and np.array_equal(b.slot_mapping, m["slot_mapping"])
    assert b.context_lens.tolist() == [0, 1, 16, 17]
    assert np.array_equal(b.block_tables, m["block_tables"])


def test_shared_prefix_cow_counts():
    # as stated: 1024 = 64 x 16, the prompt's last block is full -> no copies
    assert build_batch(workloads.make("4")).cow_pairs.shape == (0, 2)
    # prompt 1016: 63 full blocks + 1 half block shared by 8 samples; the first
    # append of 7 samples copies it, the last sample owns it alone
    b = build_batch(workloads.make("4cow"))
    assert b.cow_pairs.shape == (32 * 7, 2)
    srcs = b.cow_pairs[:, 0]
    assert len(set(srcs.tolist())) == 32          # one shared partial block per prompt
    assert len(set(b.cow_pairs[:, 1].tolist())) == 32 * 7
    assert not set(srcs.tolist()) & set(b.cow_pairs[:, 1].tolist())


def test_internal_fragmentation_bounded():
    wl = workloads.make("3")
    b = build_batch(wl)
    for i, L in enumerate(b.context_lens):
        nblk = -(-int(L) // wl.block_size)
        assert nblk * wl.block_size - L < wl.block_size


def test_fork_free_and_exhaustion():
    a = BlockAllocator(4, 16)
    s = a.new_sequence(20)                 # 2 blocks
    c = a.fork(s)
    assert all(a.refcount(x) == 2 for x in a.block_table(s))
    slot, cow = a.append_slot(c)           # position 20: last block shared -> copy
    assert cow is not None and cow[0] == a.block_table(s)[1]
    assert a.block_table(c)[1] == cow[1]
    a.free(s)                              # s's private second block returns
    assert a.num_free == 2
    a.free(c)
    assert a.num_free == 4
    with pytest.raises(PoolExhausted):
        a.new_sequence(16 * 5)
    a2 = BlockAllocator(1, 16)
    t = a2.new_sequence(16)
    with pytest.raises(PoolExhausted):
        a2.append_slot(t)
