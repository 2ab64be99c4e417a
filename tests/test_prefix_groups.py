"""Host logic of shared-prefix decode: grouping the sequences of a batch by the
physical blocks their tables share (no GPU)."""
import numpy as np
import pytest

import workloads
from paged_kv_cache_388_b200.batch import build_batch, shared_prefix_groups


def _check_invariants(bt, lens, bs, gs, gb):
    n = len(lens)
    assert gs[0] == 0 and gs[-1] == n and np.all(np.diff(gs) >= 1)
    assert len(gb) == len(gs) - 1
    for j in range(len(gb)):
        s0, s1, p = gs[j], gs[j + 1], int(gb[j])
        if s1 - s0 == 1:
            assert p == 0
        for s in range(s0, s1):
            assert p * bs <= lens[s]                       # shared blocks are full for every member
            assert np.array_equal(bt[s, :p], bt[s0, :p])  # and hold the first member's ids


@pytest.mark.parametrize("cfg,shared", [("4s", 8), ("4cows", 7), ("4", 64), ("4cow", 63)])
def test_parallel_sampling_groups(cfg, shared):
    wl = workloads.make(cfg)
    b = build_batch(wl)
    gs, gb = shared_prefix_groups(b.block_tables, b.context_lens, wl.block_size)
    # one group per prompt, its samples sharing the prompt's full blocks; the
    # copy-on-write variant's half-filled last prompt block is private after
    # the first append, so it is not shared
    assert gs.tolist() == list(range(0, wl.num_seqs + 1, wl.samples))
    assert gb.tolist() == [shared] * wl.num_prompts
    _check_invariants(b.block_tables, b.context_lens, wl.block_size, gs, gb)


def test_no_sharing_gives_singletons():
    wl = workloads.make("3s")
    b = build_batch(wl)
    gs, gb = shared_prefix_groups(b.block_tables, b.context_lens, wl.block_size)
    assert gs.tolist() == list(range(wl.num_seqs + 1))
    assert not gb.any()


def test_divergence_and_threshold():
    bs = 16
    bt = np.array([[5, 6, 7, 8, 9],
                   [5, 6, 7, 8, 1],
                   [5, 6, 2, 3, 4],     # diverges after two blocks
                   [10, 11, 12, 13, 14],
                   [10, 11, 12, 13, 15]], dtype=np.int32)
    lens = np.array([80, 70, 75, 66, 65], dtype=np.int32)
    gs, gb = shared_prefix_groups(bt, lens, bs)
    # greedy: sequence 2 still shares two blocks, so the group keeps it with 2
    assert gs.tolist() == [0, 3, 5] and gb.tolist() == [2, 4]
    _check_invariants(bt, lens, bs, gs, gb)
    gs, gb = shared_prefix_groups(bt, lens, bs, min_shared_blocks=3)
    assert gs.tolist() == [0, 2, 3, 5] and gb.tolist() == [4, 0, 4]
    _check_invariants(bt, lens, bs, gs, gb)


def test_partially_filled_shared_block_is_not_counted():
    bs = 16
    bt = np.array([[3, 4, 9], [3, 4, 9]], dtype=np.int32)
    lens = np.array([40, 40], dtype=np.int32)   # blocks 3 and 4 are full, block 9 holds 8 tokens
    gs, gb = shared_prefix_groups(bt, lens, bs)
    assert gs.tolist() == [0, 2] and gb.tolist() == [2]
    lens = np.array([40, 30], dtype=np.int32)   # the second member filled one block only
    gs, gb = shared_prefix_groups(bt, lens, bs)
    assert gb.tolist() == [1]
    _check_invariants(bt, lens, bs, gs, gb)
