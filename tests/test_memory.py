"""Memory accounting (host only): the pages' worked examples and the bound
that paging wastes less than one block per sequence."""
import numpy as np
import pytest

import workloads
from oracle import alloc_model
from oracle_pins import golden
from paged_kv_cache_388_b200.batch import build_batch
from paged_kv_cache_388_b200.memory import paged_usage, pool_usage, reserved_usage, waste_report


def test_preallocation_worked_example():
    g = golden("preallocation_waste.json")
    for case in g["cases"]:
        r = reserved_usage([case["used"]], g["max_len"])
        pct = 100.0 * r["waste_frac"]
        # the page truncates: exact value lies in [printed, printed + resolution)
        assert case["printed_pct"] <= pct < case["printed_pct"] + case["printed_resolution"], pct


def test_block_count_example_waste():
    g = golden("block_count_worked_example.json")
    p = paged_usage([g["tokens"]], g["block_size"])
    assert p["slots"] == g["blocks"] * g["block_size"]
    assert p["slots"] - p["tokens"] == g["block_size"] - g["tokens_in_last_block"]


@pytest.mark.parametrize("cfg", ["2", "3", "5"])
def test_paged_waste_below_one_block_per_sequence(cfg):
    wl = workloads.make(cfg)
    lens = wl.seq_context_lens()
    p = paged_usage(lens, wl.block_size)
    blocks = sum(alloc_model.blocks_needed(L, wl.block_size) for L in lens)
    assert p["slots"] == blocks * wl.block_size            # plain definition
    assert p["slots"] - p["tokens"] < len(lens) * wl.block_size


def test_report_on_config3_against_a_4096_reservation():
    wl = workloads.make("3")
    rep = waste_report(wl.seq_context_lens(), wl.block_size, 4096)
    assert rep["paged"]["waste_frac"] < 0.04              # the pages: under 4 %
    assert rep["reserved"]["waste_frac"] > 0.6            # the pages: 60-80 % for reservation
    assert rep["slot_ratio"] > 3


def test_pool_usage_counts_shared_blocks_once():
    wl = workloads.make("4s")
    b = build_batch(wl)
    u = pool_usage(b.allocator)
    # 2 prompts x 8 samples share 8 prompt blocks each: logical tokens exceed slots held
    assert u["tokens_logical"] > u["slots"]
    assert u["blocks"] == int(np.count_nonzero([b.allocator.refcount(i) for i in range(wl.num_blocks)]))
