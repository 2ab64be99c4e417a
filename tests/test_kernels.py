"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

reshape_and_cache and copy_blocks are compared byte for byte over the whole
pool; decode outputs element by element with |gpu - ref| <= atol + rtol*|ref|,
(atol, rtol) = (2e-3, 1e-2) for fp16/bf16 and (1e-5, 1e-5) for fp32.
"""
import numpy as np
import pytest
import torch

import workloads
from gpu_harness import assert_close, device_inputs, gpu_step, oracle_step, raw_cpu
from paged_kv_cache_388_b200.batch import build_batch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_388_b200 import _lib
    assert _lib.pa_get_device_error() == 0
    return _lib


def _check_workload(lib, wl, kv_split_tokens=0, rows=None):
    vals = workloads.values(wl)
    batch = build_batch(wl)
    d = device_inputs(wl, vals, batch)
    out = gpu_step(lib, wl, batch, d, kv_split_tokens)
    torch.cuda.synchronize()
    assert lib.pa_get_device_error() == 0
    kp, vp, ref = oracle_step(wl, vals, rows=rows)
    assert np.array_equal(raw_cpu(d["k_cache"]), kp), "K pool differs from the oracle"
    assert np.array_equal(raw_cpu(d["v_cache"]), vp), "V pool differs from the oracle"
    err = assert_close(out, ref, wl.dtype, rows=rows, what=wl.name)
    return out, ref, err


@pytest.fixture(params=["auto", "simt"])
def decode_kernel(request, monkeypatch):
    """Run with the library's default decode kernel (tensor cores for 16-bit
    caches) and with the CUDA-core kernel forced."""
    if request.param == "simt":
        monkeypatch.setenv("PA_DECODE_KERNEL", "simt")
    else:
        monkeypatch.delenv("PA_DECODE_KERNEL", raising=False)
    return request.param


@pytest.fixture(params=["auto", "pp5d", "tc64", "mma"])
def chunk_kernel(request, monkeypatch):
    """Chunked-query rows through the default kernel (tcgen05 ping-pong over
    128-key tiles at head_dim 128), the same kernel with one 5-D K/V box per
    block instead of two 2-D boxes, the tcgen05 kernel over 64-key tiles and
    the mma.sync kernel."""
    monkeypatch.delenv("PA_CHUNK_PP_BOXES", raising=False)
    if request.param == "auto":
        monkeypatch.delenv("PA_CHUNK_KERNEL", raising=False)
    elif request.param == "pp5d":
        monkeypatch.delenv("PA_CHUNK_KERNEL", raising=False)
        monkeypatch.setenv("PA_CHUNK_PP_BOXES", "5d")
    else:
        monkeypatch.setenv("PA_CHUNK_KERNEL", request.param)
    return request.param


@pytest.mark.parametrize("split", [0, 32, 1 << 20], ids=["policy", "split32", "nosplit"])
@pytest.mark.parametrize("cfg", workloads.SMALL_CONFIGS)
def test_small_config_parity(lib, cfg, split, decode_kernel):
    _check_workload(lib, workloads.make(cfg), kv_split_tokens=split)


def _full_rows(wl):
    """Every query row, except the chunked-prefill rows of the long mixed
    batches, whose fp64 reference costs ~0.27 GFLOP a row: of those, the first
    and last token of every 32-token span (the query tiles of the tensor-core
    chunk kernel hold 32 tokens x 4 heads) and every 8th token.  Every decode
    row is always compared."""
    tq = wl.num_q_tokens
    if wl.kind != "mixed" or max(wl.query_lens) <= 64:
        return None
    rows, pos = set(), 0
    for q in wl.query_lens:
        if q == 1:
            rows.add(pos)
        else:
            for t in range(q):
                if t % 8 == 0 or t % 32 in (0, 31) or t == q - 1:
                    rows.add(pos + t)
        pos += q
    assert max(rows) < tq
    return sorted(rows)


@pytest.mark.parametrize("cfg", workloads.FULL_CONFIGS)
def test_full_config_parity(lib, cfg):
    """The full-size configurations in the launch configuration the benchmark
    times (library partition policy), every row compared with the oracle."""
    wl = workloads.make(cfg)
    _check_workload(lib, wl, rows=_full_rows(wl))


def test_chunk_mixed_8k(lib):
    """Four 512-token causal chunks over 8192-token prefixes plus two decode
    rows (config 5's chunk shape at half the prefix): every chunk row."""
    wl = workloads.mixed_workload("chunk_mixed_8k", 4242, 2, 1000, 2000, 4, 8192, 512, 32, 8, 128,
                                  16, "bf16")
    _check_workload(lib, wl)


def test_split_agrees_with_nosplit(lib, decode_kernel):
    wl = workloads.make("3s")
    vals = workloads.values(wl)
    batch = build_batch(wl)
    outs = []
    for split in (16, 64, 1 << 20):
        d = device_inputs(wl, vals, batch)
        outs.append(gpu_step(lib, wl, batch, d, split).float())
    for o in outs[:-1]:
        # two bf16 roundings of nearly equal fp32 values differ by at most 1 ulp
        # of the larger one (2^-7 of it covers an ulp in any binade)
        diff = (o - outs[-1]).abs()
        assert torch.all(diff <= 2.0 ** -7 * torch.maximum(o.abs(), outs[-1].abs()) + 1e-6), diff.max()


@pytest.mark.parametrize("bs", [16, 32])
@pytest.mark.parametrize("H,Hk,D,dtype", [(32, 8, 128, "bf16"), (8, 4, 64, "f16"),
                                          (32, 2, 128, "bf16"), (4, 4, 64, "f32"),
                                          (16, 2, 64, "f32")])
def test_edge_lengths(lib, H, Hk, D, dtype, bs, decode_kernel):
    lens = [0, 1, 15, 16, 17, 31, 32, 33, 513, 4096]
    wl = workloads.decode_workload(f"edge_{H}_{Hk}_{D}_{dtype}_{bs}", 3100, lens, H, Hk, D, bs, dtype)
    out, ref, _ = _check_workload(lib, wl, kv_split_tokens=64)
    assert torch.count_nonzero(out[0]) == 0  # empty context -> zeros
    _check_workload(lib, wl, kv_split_tokens=0)


@pytest.mark.parametrize("dtype,D,bs", [("bf16", 128, 16), ("f16", 64, 32), ("f32", 64, 16),
                                        ("bf16", 64, 32)])
def test_chunked_rows(lib, dtype, D, bs, decode_kernel, chunk_kernel):
    wl = workloads.mixed_workload(f"chunk_{dtype}_{D}_{bs}", 3200, 2, 100, 900, 3, 150, 37,
                                  16, 4, D, bs, dtype)
    _check_workload(lib, wl)


def test_chunk_group_eight(lib, chunk_kernel):
    wl = workloads.mixed_workload("chunk_g8", 3300, 1, 300, 400, 2, 64, 20, 64, 8, 128, 16, "bf16")
    _check_workload(lib, wl)


def test_chunk_whole_prompt(lib, chunk_kernel):
    # a chunk that is the whole context (L == Q): row t sees keys 0..t
    wl = workloads.mixed_workload("chunk_full", 3400, 1, 5, 9, 2, 0, 77, 32, 8, 128, 16, "bf16")
    _check_workload(lib, wl)


@pytest.mark.parametrize("G,bs,dtype", [(1, 16, "bf16"), (2, 32, "f16"), (8, 32, "bf16"),
                                        (16, 16, "bf16"), (4, 16, "f16")])
def test_chunk_shapes(lib, G, bs, dtype, chunk_kernel):
    # groups 1..16, both block sizes, chunk lengths that leave ragged tiles
    Hk = 2
    wl = workloads.mixed_workload(f"chunk_shapes_{G}_{bs}_{dtype}", 3500 + G, 2, 50, 400, 3, 131, 45,
                                  G * Hk, Hk, 128, bs, dtype)
    _check_workload(lib, wl)


def _ws(lib, n, split=0, H=8, Hk=2, D=128, bs=16, max_ctx=64):
    size = lib.pa_decode_workspace_size(n, H, Hk, D, bs, max_ctx, split)
    return torch.empty(max(size, 16), dtype=torch.uint8, device="cuda")


def _tiny_decode(lib, lens=(20, 40), dtype=torch.bfloat16, bs=16):
    torch.manual_seed(0)
    H, Hk, D = 8, 2, 128
    nb = 16
    kc = torch.randn(nb, Hk, bs, D, device="cuda").to(dtype)
    vc = torch.randn(nb, Hk, bs, D, device="cuda").to(dtype)
    q = torch.randn(len(lens), H, D, device="cuda").to(dtype)
    bt = torch.arange(len(lens) * 4, dtype=torch.int32, device="cuda").reshape(len(lens), 4) % nb
    cl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    return kc, vc, q, bt, cl


def test_bad_block_id_sets_error_and_zeroes_row(lib, decode_kernel):
    kc, vc, q, bt, cl = _tiny_decode(lib)
    bt[1, 1] = 10_000
    out = torch.full_like(q, 7.0)
    lib.pa_decode(out, q, kc, vc, bt, cl, 0.1, kv_split_tokens=1 << 20, workspace=_ws(lib, 2))
    code = lib.pa_get_device_error()
    assert code & lib.PA_DEVERR_BLOCK_ID
    assert torch.count_nonzero(out[1]) == 0
    assert torch.all(torch.isfinite(out[0].float())) and torch.count_nonzero(out[0]) > 0
    assert lib.pa_get_device_error() == 0  # cleared


def test_bad_block_id_split_path(lib, decode_kernel):
    kc, vc, q, bt, cl = _tiny_decode(lib, lens=(20, 60))
    bt[1, 3] = -5
    ws = torch.empty(lib.pa_decode_workspace_size(2, 8, 2, 128, 16, 64, 16), dtype=torch.uint8,
                     device="cuda")
    out = torch.full_like(q, 7.0)
    lib.pa_decode(out, q, kc, vc, bt, cl, 0.1, kv_split_tokens=16, workspace=ws)
    assert lib.pa_get_device_error() & lib.PA_DEVERR_BLOCK_ID
    assert torch.count_nonzero(out[1]) == 0


def test_bad_context_len(lib, decode_kernel):
    kc, vc, q, bt, cl = _tiny_decode(lib)
    cl[0] = 4 * 16 + 1  # beyond max_blocks_per_seq * block_size
    out = torch.full_like(q, 7.0)
    lib.pa_decode(out, q, kc, vc, bt, cl, 0.1, workspace=_ws(lib, 2))
    assert lib.pa_get_device_error() & lib.PA_DEVERR_CONTEXT_LEN
    assert torch.count_nonzero(out[0]) == 0


def test_reshape_padding_and_bad_slot(lib):
    Hk, D, bs, nb = 2, 128, 16, 8
    kc = torch.randn(nb, Hk, bs, D, device="cuda").to(torch.bfloat16)
    vc = torch.randn(nb, Hk, bs, D, device="cuda").to(torch.bfloat16)
    k0, v0 = kc.clone(), vc.clone()
    key = torch.randn(3, Hk, D, device="cuda").to(torch.bfloat16)
    val = torch.randn(3, Hk, D, device="cuda").to(torch.bfloat16)
    slots = torch.tensor([5 * 16 + 3, -1, nb * bs + 7], dtype=torch.int64, device="cuda")
    lib.pa_reshape_and_cache(key, val, kc, vc, slots)
    assert lib.pa_get_device_error() & lib.PA_DEVERR_SLOT
    k0[5, :, 3] = key[0]
    v0[5, :, 3] = val[0]
    assert torch.equal(kc, k0) and torch.equal(vc, v0)


def test_copy_blocks_random_pairs(lib):
    Hk, D, bs, nb = 8, 128, 16, 64
    for dt in (torch.bfloat16, torch.float32):
        kc = torch.randn(nb, Hk, bs, D, device="cuda").to(dt)
        vc = torch.randn(nb, Hk, bs, D, device="cuda").to(dt)
        perm = torch.randperm(nb)
        src, dst = perm[:20], perm[20:40]
        pairs = torch.stack([src, dst], 1).to(torch.int64).cuda()
        k0, v0 = kc.clone(), vc.clone()
        lib.pa_copy_blocks(kc, vc, pairs)
        k0[dst] = k0[src]
        v0[dst] = v0[src]
        assert torch.equal(kc, k0) and torch.equal(vc, v0)
        bad = torch.tensor([[0, nb]], dtype=torch.int64, device="cuda")
        lib.pa_copy_blocks(kc, vc, bad)
        assert lib.pa_get_device_error() & lib.PA_DEVERR_BLOCK_ID
        assert torch.equal(kc, k0)


def test_host_argument_errors(lib):
    kc, vc, q, bt, cl = _tiny_decode(lib, lens=(20, 60))
    out = torch.empty_like(q)
    with pytest.raises(lib.PAError) as e:  # split needs a workspace
        lib.pa_decode(out, q, kc, vc, bt, cl, 0.1, kv_split_tokens=16, workspace=None)
    assert e.value.status == -3
    small = torch.empty(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(lib.PAError) as e:
        lib.pa_decode(out, q, kc, vc, bt, cl, 0.1, kv_split_tokens=16, workspace=small)
    assert e.value.status == -3
    # unsupported head_dim: call the entry point directly (96 is not in {64, 128})
    rc = lib.library().pa_decode(out.data_ptr(), q.data_ptr(), kc.data_ptr(), vc.data_ptr(),
                                 bt.data_ptr(), 4, cl.data_ptr(), None, 2, 2, 1, 8, 2, 96, 16, 16,
                                 0.1, 0, 0, 2, None, 0, None)
    assert rc == -2
    # misaligned q pointer
    rc = lib.library().pa_decode(out.data_ptr(), q.data_ptr() + 2, kc.data_ptr(), vc.data_ptr(),
                                 bt.data_ptr(), 4, cl.data_ptr(), None, 2, 2, 1, 8, 2, 128, 16, 16,
                                 0.1, 0, 0, 2, None, 0, None)
    assert rc == -1
    # out aliasing q
    rc = lib.library().pa_decode(q.data_ptr(), q.data_ptr(), kc.data_ptr(), vc.data_ptr(),
                                 bt.data_ptr(), 4, cl.data_ptr(), None, 2, 2, 1, 8, 2, 128, 16, 16,
                                 0.1, 0, 0, 2, None, 0, None)
    assert rc == -1
    assert lib.pa_get_device_error() == 0


def test_empty_calls_are_noops(lib):
    kc, vc, q, bt, cl = _tiny_decode(lib)
    k0 = kc.clone()
    e = torch.empty(0, 2, 128, device="cuda", dtype=torch.bfloat16)
    lib.pa_reshape_and_cache(e, e, kc, vc, torch.empty(0, dtype=torch.int64, device="cuda"))
    lib.pa_copy_blocks(kc, vc, torch.empty(0, 2, dtype=torch.int64, device="cuda"))
    assert torch.equal(kc, k0)
    assert lib.pa_get_device_error() == 0


def test_nan_in_unused_slots_does_not_leak(lib, decode_kernel):
    """Slots past a sequence's length may hold anything; NaN there must not
    reach the output."""
    kc, vc, q, bt, cl = _tiny_decode(lib, lens=(20, 37))
    nan = torch.tensor(float("nan"), dtype=kc.dtype, device="cuda")
    ref_out = torch.empty_like(q)
    ref_bal = torch.empty_like(q)
    ws = _ws(lib, 2)
    lib.pa_decode(ref_out, q, kc, vc, bt, cl, 0.1, kv_split_tokens=1 << 20, workspace=ws)
    # the balanced partition sums in another order: its own reference
    lib.pa_decode(ref_bal, q, kc, vc, bt, cl, 0.1, workspace=ws)
    kc[bt[0, 1], :, 4:] = nan  # seq 0: tokens 20.. of block 1 are unused
    vc[bt[0, 1], :, 4:] = nan
    kc[bt[1, 2], :, 5:] = nan  # seq 1: tokens 37.. of block 2
    vc[bt[1, 2], :, 5:] = nan
    out = torch.empty_like(q)
    lib.pa_decode(out, q, kc, vc, bt, cl, 0.1, kv_split_tokens=1 << 20, workspace=ws)
    assert lib.pa_get_device_error() == 0
    assert torch.equal(out, ref_out)
    lib.pa_decode(out, q, kc, vc, bt, cl, 0.1, workspace=ws)  # balanced partition
    assert lib.pa_get_device_error() == 0
    assert torch.equal(out, ref_bal)
