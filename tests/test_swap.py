"""GPU parity of pa_swap_blocks (block moves between a device pool and a
page-locked host pool) against the CPU oracle: byte-exact over the whole
destination pool, the source pool untouched, and a swap-out / swap-in round
trip restoring the device blocks."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_388_b200 import _lib
    assert _lib.pa_get_device_error() == 0
    return _lib


def _pool(nb, Hk, bs, D, dtype, seed, where):
    g = torch.Generator().manual_seed(seed)
    t = torch.randn((nb, Hk, bs, D), generator=g).to(workloads.torch_dtype(dtype))
    if where == "cuda":
        return t.cuda()
    return t.pin_memory()


def _raw(t):
    return workloads.to_numpy_raw(t.cpu())


@pytest.mark.parametrize("dtype,Hk,bs,D", [("bf16", 8, 16, 128), ("f16", 4, 32, 64),
                                           ("f32", 2, 16, 64), ("bf16", 8, 32, 128)])
@pytest.mark.parametrize("direction", ["out", "in", "device_to_device", "host_to_host"])
def test_swap_matches_oracle(lib, dtype, Hk, bs, D, direction):
    src_where, dst_where = {"out": ("cuda", "host"), "in": ("host", "cuda"),
                            "device_to_device": ("cuda", "cuda"),
                            "host_to_host": ("host", "host")}[direction]
    ns, nd = 300, 170
    src_k = _pool(ns, Hk, bs, D, dtype, 1, src_where)
    src_v = _pool(ns, Hk, bs, D, dtype, 2, src_where)
    dst_k = _pool(nd, Hk, bs, D, dtype, 3, dst_where)
    dst_v = _pool(nd, Hk, bs, D, dtype, 4, dst_where)
    rng = np.random.default_rng(5)
    pairs = np.stack([rng.permutation(ns)[:123], rng.permutation(nd)[:123]], 1).astype(np.int64)
    want_k, want_v = _raw(dst_k).copy(), _raw(dst_v).copy()
    src_k0, src_v0 = _raw(src_k).copy(), _raw(src_v).copy()
    oracle.swap_blocks(want_k, want_v, src_k0, src_v0, pairs, dtype)
    mapping = torch.from_numpy(pairs)
    mapping = mapping.cuda() if direction != "host_to_host" else mapping.pin_memory()
    lib.pa_swap_blocks(dst_k, dst_v, src_k, src_v, mapping)
    torch.cuda.synchronize()
    assert lib.pa_get_device_error() == 0
    assert np.array_equal(_raw(dst_k), want_k) and np.array_equal(_raw(dst_v), want_v)
    assert np.array_equal(_raw(src_k), src_k0) and np.array_equal(_raw(src_v), src_v0)


def test_round_trip_through_the_host_tier(lib):
    from paged_kv_cache_388_b200.session import PagedKVCache
    wl = workloads.make("3s")
    vals = workloads.values(wl)
    cache = PagedKVCache(wl.num_blocks, wl.num_kv_heads, wl.head_dim, wl.block_size,
                         k_cache=vals["k_pool"].cuda(), v_cache=vals["v_pool"].cuda())
    k0, v0 = cache.k_cache.clone(), cache.v_cache.clone()
    host_k, host_v = cache.host_pool(64)
    dev_blocks = torch.from_numpy(np.random.default_rng(9).permutation(wl.num_blocks)[:64])
    out_map = torch.stack([dev_blocks, torch.arange(64)], 1).cuda()
    cache.swap_out(host_k, host_v, out_map)
    cache.k_cache[dev_blocks.cuda()] = 0      # the blocks are handed to other sequences
    cache.v_cache[dev_blocks.cuda()] = 0
    cache.swap_in(host_k, host_v, out_map.flip(1).contiguous())
    torch.cuda.synchronize()
    assert lib.pa_get_device_error() == 0
    assert torch.equal(cache.k_cache, k0) and torch.equal(cache.v_cache, v0)


def test_bad_block_ids_are_skipped(lib):
    src_k = _pool(8, 2, 16, 64, "bf16", 1, "cuda")
    src_v = _pool(8, 2, 16, 64, "bf16", 2, "cuda")
    dst_k = _pool(4, 2, 16, 64, "bf16", 3, "host")
    dst_v = _pool(4, 2, 16, 64, "bf16", 4, "host")
    d0k, d0v = dst_k.clone(), dst_v.clone()
    mapping = torch.tensor([[1, 0], [9, 1], [2, -1], [3, 2]], dtype=torch.int64, device="cuda")
    lib.pa_swap_blocks(dst_k, dst_v, src_k, src_v, mapping)
    assert lib.pa_get_device_error() & lib.PA_DEVERR_BLOCK_ID
    assert torch.equal(dst_k[0], src_k[1].cpu()) and torch.equal(dst_v[2], src_v[3].cpu())
    assert torch.equal(dst_k[1], d0k[1]) and torch.equal(dst_v[3], d0v[3])


def test_pageable_host_memory_is_rejected(lib):
    src_k = _pool(4, 2, 16, 64, "bf16", 1, "cuda")
    src_v = _pool(4, 2, 16, 64, "bf16", 2, "cuda")
    pageable_k = torch.empty((4, 2, 16, 64), dtype=torch.bfloat16)
    pageable_v = torch.empty((4, 2, 16, 64), dtype=torch.bfloat16)
    mapping = torch.tensor([[0, 0]], dtype=torch.int64, device="cuda")
    with pytest.raises(ValueError):
        lib.pa_swap_blocks(pageable_k, pageable_v, src_k, src_v, mapping)
    # the C entry point itself refuses before launching anything
    raw = lib.library()
    rc = raw.pa_swap_blocks(ctypes.c_void_p(pageable_k.data_ptr()),
                            ctypes.c_void_p(pageable_v.data_ptr()),
                            ctypes.c_void_p(src_k.data_ptr()), ctypes.c_void_p(src_v.data_ptr()),
                            ctypes.c_void_p(mapping.data_ptr()), 1, 2, 64, 16, 4, 4, 2, None)
    assert rc == -1
    torch.cuda.synchronize()
    assert lib.pa_get_device_error() == 0


def test_empty_mapping_is_a_noop(lib):
    k = _pool(2, 2, 16, 64, "bf16", 1, "cuda")
    h = _pool(2, 2, 16, 64, "bf16", 2, "host")
    h0 = h.clone()
    lib.pa_swap_blocks(h, h, k, k, torch.empty((0, 2), dtype=torch.int64, device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(h, h0)
