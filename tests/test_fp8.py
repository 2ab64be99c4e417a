"""GPU parity of the FP8 (E4M3) KV cache against the CPU oracle.

pa_reshape_and_cache_fp8 must write exactly the oracle's codes over the whole
pool (the quantiser is integer output decided by binary32 arithmetic, done in
the same precision on both sides); pa_decode_fp8 must match the oracle's
attention over the dequantised cache within the decode tolerance.  The
history already in the pool is quantised on the host (torch's float8
conversion of the binary32 quotient, which saturates nothing at these
scales) so that both sides start from the same codes.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_harness import assert_close
from paged_kv_cache_388_b200.batch import build_batch, shared_prefix_groups, staged_blocks_needed

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_388_b200 import _lib
    assert _lib.pa_get_device_error() == 0
    return _lib


def _scale(*ts):
    amax = max(float(t.float().abs().max()) for t in ts)
    return float(np.float32(amax / 448.0 * 1.25))


def _quant(t, s):
    return (t.float() / torch.tensor(s, dtype=torch.float32)).to(torch.float8_e4m3fn).view(torch.uint8)


def _run(lib, wl, rows=None, q_mul=1.0, staged=None, expect_err=0):
    """One step over an FP8 cache; mixed batches (chunk rows) go through
    pa_decode_fp8_rows with `staged` blocks of staging (default: exactly what
    the batch needs).  With expect_err the device error word must hold those
    bits and every compared row is either the oracle's or zero."""
    vals = workloads.values(wl)
    batch = build_batch(wl)
    mixed = batch.query_start_loc is not None and batch.max_query_len > 1
    ks = _scale(vals["k_pool"], vals["new_key"])
    vs = _scale(vals["v_pool"], vals["new_value"])
    kp, vp = _quant(vals["k_pool"], ks), _quant(vals["v_pool"], vs)
    q = (vals["q"].float() * q_mul).to(vals["q"].dtype)
    dev = "cuda"
    k8, v8 = kp.to(dev), vp.to(dev)
    key, value = vals["new_key"].to(dev), vals["new_value"].to(dev)
    slot = torch.from_numpy(batch.slot_mapping).to(dev)
    bt = torch.from_numpy(batch.block_tables).to(dev)
    cl = torch.from_numpy(batch.context_lens).to(dev)
    cow = torch.from_numpy(np.ascontiguousarray(batch.cow_pairs)).to(dev)
    if cow.shape[0]:
        lib.pa_copy_blocks(k8, v8, cow)
    lib.pa_reshape_and_cache_fp8(key, value, k8, v8, slot, ks, vs)
    out = torch.full_like(q, float("nan"), device=dev)
    if mixed:
        if staged is None:
            staged = staged_blocks_needed(batch.query_start_loc, batch.context_lens, wl.block_size)
        size = lib.pa_decode_fp8_rows_workspace_size(batch.num_seqs, wl.num_heads, wl.num_kv_heads,
                                                     wl.head_dim, wl.block_size,
                                                     batch.max_context_len,
                                                     batch.block_tables.shape[1], staged)
        ws = torch.empty(max(size, 16), dtype=torch.uint8, device=dev)
        lib.pa_decode_fp8(out, q.to(dev), k8, v8, bt, cl, wl.scale, ks, vs,
                          max_context_len=batch.max_context_len, workspace=ws,
                          query_start_loc=torch.from_numpy(batch.query_start_loc).to(dev),
                          max_query_len=batch.max_query_len, staged_blocks=staged)
    else:
        size = lib.pa_decode_workspace_size(batch.num_seqs, wl.num_heads, wl.num_kv_heads,
                                            wl.head_dim, wl.block_size, batch.max_context_len, 0)
        ws = torch.empty(max(size, 16), dtype=torch.uint8, device=dev)
        lib.pa_decode_fp8(out, q.to(dev), k8, v8, bt, cl, wl.scale, ks, vs,
                          max_context_len=batch.max_context_len, workspace=ws)
    torch.cuda.synchronize()
    assert lib.pa_get_device_error() == expect_err
    # the oracle, from the same starting codes
    kpn, vpn = kp.numpy().copy(), vp.numpy().copy()
    if batch.cow_pairs.shape[0]:
        oracle.copy_blocks(kpn, vpn, batch.cow_pairs, "fp8")
    oracle.reshape_and_cache_fp8(kpn, vpn, workloads.to_numpy_raw(vals["new_key"]),
                                 workloads.to_numpy_raw(vals["new_value"]), wl.dtype,
                                 batch.slot_mapping, ks, vs)
    assert np.array_equal(k8.cpu().numpy(), kpn), "K codes differ from the oracle"
    assert np.array_equal(v8.cpu().numpy(), vpn), "V codes differ from the oracle"
    ref = oracle.decode_fp8(workloads.to_numpy_raw(q), wl.dtype, kpn, vpn, ks, vs,
                            batch.block_tables, batch.context_lens, wl.scale,
                            query_start_loc=batch.query_start_loc if mixed else None, rows=rows)
    if expect_err:
        return out, ref
    assert_close(out, ref, "bf16", rows=rows, what=wl.name + " fp8")
    return out


@pytest.mark.parametrize("cfg", ["3s", "3s32", "2s", "4s", "4cows"])
def test_small_configs(lib, cfg):
    _run(lib, workloads.make(cfg))


@pytest.mark.parametrize("cfg", ["2", "3"])
def test_full_configs(lib, cfg):
    """Full-size batches in the benchmark's launch configuration, every row."""
    _run(lib, workloads.make(cfg))


@pytest.mark.parametrize("q_mul", [1000.0, 1e-3, 3e4])
def test_bf16_query_range(lib, q_mul):
    """bf16 q rows are brought into fp16 range by a power of two per head."""
    _run(lib, workloads.make("3s"), q_mul=q_mul)


@pytest.mark.parametrize("H,Hk,D,bs,dtype", [(32, 8, 128, 16, "bf16"), (8, 4, 64, 32, "f16"),
                                             (32, 2, 128, 32, "bf16"), (4, 4, 64, 16, "f16")])
def test_edge_lengths(lib, H, Hk, D, bs, dtype):
    lens = [0, 1, 15, 16, 17, 31, 32, 33, 513, 2049]
    wl = workloads.decode_workload(f"fp8_edge_{H}_{Hk}_{D}_{bs}_{dtype}", 3300, lens, H, Hk, D, bs,
                                   dtype)
    _run(lib, wl)


def test_host_argument_errors(lib):
    q = torch.randn(2, 8, 128, device="cuda").to(torch.bfloat16)
    k8 = torch.zeros(4, 2, 16, 128, dtype=torch.uint8, device="cuda")
    bt = torch.zeros(2, 2, dtype=torch.int32, device="cuda")
    cl = torch.tensor([3, 5], dtype=torch.int32, device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(lib.PAError) as e:
        lib.pa_decode_fp8(torch.empty_like(q), q, k8, k8, bt, cl, 0.1, 0.0, 1.0, workspace=ws)
    assert e.value.status == -1  # a scale must be positive
    with pytest.raises(lib.PAError) as e:
        q32 = q.float()
        lib.pa_decode_fp8(torch.empty_like(q32), q32, k8, k8, bt, cl, 0.1, 1.0, 1.0, workspace=ws)
    assert e.value.status == -2  # q/out must be fp16 or bf16
    key = torch.randn(1, 2, 128, device="cuda")
    with pytest.raises(lib.PAError) as e:
        lib.pa_reshape_and_cache_fp8(key, key, k8, k8, torch.zeros(1, dtype=torch.int64, device="cuda"),
                                     float("inf"), 1.0)
    assert e.value.status == -1
    torch.cuda.synchronize()
    assert lib.pa_get_device_error() == 0


def test_saturation_and_bad_slot(lib):
    """Magnitudes beyond 448 * scale store +-448; a slot past the pool is
    skipped and reported."""
    k8 = torch.zeros(2, 1, 16, 64, dtype=torch.uint8, device="cuda")
    v8 = torch.zeros_like(k8)
    key = torch.full((2, 1, 64), 1e4, device="cuda")
    key[0, 0, ::2] = -1e4
    slot = torch.tensor([3, 99], dtype=torch.int64, device="cuda")
    lib.pa_reshape_and_cache_fp8(key, key, k8, v8, slot, 1.0, 1.0)
    assert lib.pa_get_device_error() & lib.PA_DEVERR_SLOT
    row = k8[0, 0, 3].cpu()
    assert torch.all(row[::2] == 0xFE) and torch.all(row[1::2] == 0x7E)
    assert int(k8.count_nonzero()) == 64


def test_session_fp8_step(lib):
    """The session's FP8 cache: write quantises, attend decodes the codes."""
    from paged_kv_cache_388_b200.session import PagedKVCache
    wl = workloads.make("3s")
    vals = workloads.values(wl)
    batch = build_batch(wl)
    ks = _scale(vals["k_pool"], vals["new_key"])
    vs = _scale(vals["v_pool"], vals["new_value"])
    cache = PagedKVCache(wl.num_blocks, wl.num_kv_heads, wl.head_dim, wl.block_size,
                         dtype=torch.uint8, k_cache=_quant(vals["k_pool"], ks).cuda(),
                         v_cache=_quant(vals["v_pool"], vs).cuda(), kv_scales=(ks, vs))
    cache.write(vals["new_key"].cuda(), vals["new_value"].cuda(),
                torch.from_numpy(batch.slot_mapping).cuda())
    out = cache.attend(vals["q"].cuda(), torch.from_numpy(batch.block_tables).cuda(),
                       torch.from_numpy(batch.context_lens).cuda(), wl.scale,
                       max_context_len=batch.max_context_len)
    ref = _run(lib, wl)
    assert torch.equal(out, ref)


# ---- chunked-prefill rows over an FP8 cache (pa_decode_fp8_rows) ------------

@pytest.mark.parametrize("cfg", ["5s", "5s32"])
def test_chunk_rows_small(lib, cfg):
    """Decode rows and 96-token chunks over 700-token prefixes, every row."""
    _run(lib, workloads.make(cfg))


@pytest.mark.parametrize("H,Hk,D,bs,dtype", [(16, 4, 128, 16, "f16"), (8, 2, 64, 32, "bf16"),
                                             (16, 2, 64, 16, "f16")])
def test_chunk_rows_shapes(lib, H, Hk, D, bs, dtype):
    """Other groups, head_dim 64 (the mma.sync chunk kernel) and fp16 q."""
    wl = workloads.mixed_workload(f"fp8_chunk_{H}_{Hk}_{D}_{bs}_{dtype}", 3400, 2, 100, 900, 3, 150,
                                  37, H, Hk, D, bs, dtype)
    _run(lib, wl)


def _sample_rows(wl):
    batch = build_batch(wl)
    qsl = batch.query_start_loc
    rows = []
    for i in range(batch.num_seqs):
        q0, q1 = int(qsl[i]), int(qsl[i + 1])
        if q1 - q0 == 1:
            rows.append(q0)
        else:
            rows += list(range(q0, q1, 8)) + [q1 - 1]
    return sorted(set(rows))


@pytest.mark.parametrize("cfg", ["5", "5bs32"])
def test_chunk_rows_full(lib, cfg):
    """The long mixed batch over an FP8 cache: every decode row, every 8th
    chunk row and each chunk's last row."""
    wl = workloads.make(cfg)
    _run(lib, wl, rows=_sample_rows(wl))


def test_staging_overflow(lib):
    """A staging bound one block short: PA_DEVERR_STAGING (and BLOCK_ID for
    the block left out), the rows whose keys reach that block are zeros and
    every other row is the oracle's."""
    wl = workloads.make("5s")
    batch = build_batch(wl)
    need = staged_blocks_needed(batch.query_start_loc, batch.context_lens, wl.block_size)
    out, ref = _run(lib, wl, staged=need - 1,
                    expect_err=lib.PA_DEVERR_STAGING | lib.PA_DEVERR_BLOCK_ID)
    g = out.float().cpu().numpy().astype(np.float64)
    zero = np.all(g == 0.0, axis=(1, 2))
    ok = np.all(np.abs(g - ref) <= 2e-3 + 1e-2 * np.abs(ref), axis=(1, 2))
    assert np.all(zero | ok)
    assert zero.any() and ok.any()


# ---- shared prefixes over an FP8 cache (pa_decode_shared_prefix_fp8) --------

def _run_shared(lib, wl, staged=None, expect_err=0, mutate=None):
    """One step over an FP8 cache through pa_decode_shared_prefix_fp8 with the
    batch's shared-prefix groups, against the oracle's plain FP8 decode (the
    same attention).  `mutate(block_tables) -> block_tables` alters the tables
    the call and the oracle see; returns (out, ref)."""
    vals = workloads.values(wl)
    batch = build_batch(wl)
    ks = _scale(vals["k_pool"], vals["new_key"])
    vs = _scale(vals["v_pool"], vals["new_value"])
    kp, vp = _quant(vals["k_pool"], ks), _quant(vals["v_pool"], vs)
    dev = "cuda"
    k8, v8 = kp.to(dev), vp.to(dev)
    cow = torch.from_numpy(np.ascontiguousarray(batch.cow_pairs)).to(dev)
    if cow.shape[0]:
        lib.pa_copy_blocks(k8, v8, cow)
    lib.pa_reshape_and_cache_fp8(vals["new_key"].to(dev), vals["new_value"].to(dev), k8, v8,
                                 torch.from_numpy(batch.slot_mapping).to(dev), ks, vs)
    gs, gb = shared_prefix_groups(batch.block_tables, batch.context_lens, wl.block_size)
    assert int(gb.max()) > 0, "the workload must share blocks"
    bt_np = batch.block_tables if mutate is None else mutate(batch.block_tables.copy())
    if staged is None:
        staged = int(gb.sum())
    size = lib.pa_decode_shared_prefix_fp8_workspace_size(
        batch.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.block_size,
        batch.max_context_len, batch.block_tables.shape[1], gb.shape[0], staged)
    ws = torch.empty(size, dtype=torch.uint8, device=dev)
    q = vals["q"].to(dev)
    out = torch.full_like(q, float("nan"))
    lib.pa_decode_shared_prefix_fp8(out, q, k8, v8, torch.from_numpy(bt_np).to(dev),
                                    torch.from_numpy(batch.context_lens).to(dev),
                                    torch.from_numpy(gs).to(dev), torch.from_numpy(gb).to(dev),
                                    wl.scale, ks, vs, staged, max_group_size=int(np.diff(gs).max()),
                                    max_context_len=batch.max_context_len, workspace=ws)
    torch.cuda.synchronize()
    assert lib.pa_get_device_error() == expect_err
    kpn, vpn = kp.numpy().copy(), vp.numpy().copy()
    if batch.cow_pairs.shape[0]:
        oracle.copy_blocks(kpn, vpn, batch.cow_pairs, "fp8")
    oracle.reshape_and_cache_fp8(kpn, vpn, workloads.to_numpy_raw(vals["new_key"]),
                                 workloads.to_numpy_raw(vals["new_value"]), wl.dtype,
                                 batch.slot_mapping, ks, vs)
    ref = oracle.decode_fp8(workloads.to_numpy_raw(vals["q"]), wl.dtype, kpn, vpn, ks, vs, bt_np,
                            batch.context_lens, wl.scale)
    return out, ref


@pytest.mark.parametrize("prefix_kernel", ["auto", "pp", "mma"])
@pytest.mark.parametrize("cfg", ["4s", "4cows"])
def test_shared_prefix_small(lib, monkeypatch, cfg, prefix_kernel):
    """Every prefix kernel over the staged shared blocks, every row."""
    if prefix_kernel == "auto":
        monkeypatch.delenv("PA_PREFIX_KERNEL", raising=False)
    else:
        monkeypatch.setenv("PA_PREFIX_KERNEL", prefix_kernel)
    wl = workloads.make(cfg)
    out, ref = _run_shared(lib, wl)
    assert_close(out, ref, "bf16", what=wl.name + " fp8 shared-prefix")


@pytest.mark.parametrize("cfg", ["4", "4cow"])
def test_shared_prefix_full(lib, cfg):
    """Full-size parallel-sampling batches over an FP8 cache, every row."""
    wl = workloads.make(cfg)
    out, ref = _run_shared(lib, wl)
    assert_close(out, ref, "bf16", what=wl.name + " fp8 shared-prefix")


def test_shared_prefix_member_mismatch(lib):
    """A member whose table leaves its group's block: PA_DEVERR_PREFIX and a
    zero row for it, every other row the oracle's."""
    wl = workloads.make("4s")

    def mutate(bt):
        bt[2, 1] = bt[9, 1]  # sequence 2 no longer holds its group's block 1
        return bt
    out, ref = _run_shared(lib, wl, expect_err=lib.PA_DEVERR_PREFIX, mutate=mutate)
    assert torch.count_nonzero(out[2]) == 0
    keep = [i for i in range(out.shape[0]) if i != 2]
    assert_close(out, ref, "bf16", rows=keep, what="fp8 shared-prefix other members")


def test_shared_prefix_staging_overflow(lib):
    """A staging bound one block short: PA_DEVERR_STAGING (and BLOCK_ID for the
    block left out); each row is the oracle's or zeros, some of each."""
    wl = workloads.make("4s")
    batch = build_batch(wl)
    gb = shared_prefix_groups(batch.block_tables, batch.context_lens, wl.block_size)[1]
    out, ref = _run_shared(lib, wl, staged=int(gb.sum()) - 1,
                           expect_err=lib.PA_DEVERR_STAGING | lib.PA_DEVERR_BLOCK_ID)
    g = out.float().cpu().numpy().astype(np.float64)
    zero = np.all(g == 0.0, axis=(1, 2))
    ok = np.all(np.abs(g - ref) <= 2e-3 + 1e-2 * np.abs(ref), axis=(1, 2))
    assert np.all(zero | ok)
    assert zero.any() and ok.any()
