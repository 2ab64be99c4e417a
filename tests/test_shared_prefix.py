"""GPU parity of shared-prefix decode (pa_decode_shared_prefix) against the
CPU oracle.

Sharing blocks changes where keys live, not the attention, so the reference is
the oracle's plain paged decode of the same step; the shared-prefix path must
match it within the decode tolerance and must agree with pa_decode to within
fp32 rounding.  Also covered: several group shapes (group heads 1..16, head
dim 64/128, block size 16/32, fp16/bf16, member chunks), every cluster size of
the prefix kernel, members whose keys all lie in the shared prefix, groups
that do not cover the batch, and the device-side checks (a member whose table
differs in the shared range, a context shorter than the shared prefix, a bad
block id, malformed group arrays).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_harness import assert_close, device_inputs, oracle_step
from paged_kv_cache_388_b200.batch import build_batch, shared_prefix_groups

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_388_b200 import _lib
    assert _lib.pa_get_device_error() == 0
    return _lib


def _groups(batch, bs, device="cuda"):
    gs, gb = shared_prefix_groups(batch.block_tables, batch.context_lens, bs)
    return (torch.from_numpy(gs).to(device), torch.from_numpy(gb).to(device),
            int(np.diff(gs).max()))


def _prepare(lib, wl, batch, d):
    """copy_blocks + reshape_and_cache of the step (the cache the decode reads)."""
    if d["cow"].shape[0]:
        lib.pa_copy_blocks(d["k_cache"], d["v_cache"], d["cow"])
    lib.pa_reshape_and_cache(d["key"], d["value"], d["k_cache"], d["v_cache"], d["slot_mapping"])


def _shared(lib, wl, batch, d, gs, gb, max_group=0, block_tables=None, context_lens=None):
    bt = d["block_tables"] if block_tables is None else block_tables
    cl = d["context_lens"] if context_lens is None else context_lens
    out = torch.full_like(d["q"], 7.0)
    size = lib.pa_decode_shared_prefix_workspace_size(batch.num_seqs, wl.num_heads, wl.num_kv_heads,
                                                      wl.head_dim, wl.block_size,
                                                      batch.max_context_len)
    ws = torch.empty(size, dtype=torch.uint8, device="cuda")
    lib.pa_decode_shared_prefix(out, d["q"], d["k_cache"], d["v_cache"], bt, cl, gs, gb, wl.scale,
                                max_group_size=max_group, max_context_len=batch.max_context_len,
                                workspace=ws)
    return out


def _plain(lib, wl, batch, d):
    out = torch.empty_like(d["q"])
    size = lib.pa_decode_workspace_size(batch.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim,
                                        wl.block_size, batch.max_context_len, 0)
    ws = torch.empty(max(size, 16), dtype=torch.uint8, device="cuda")
    lib.pa_decode(out, d["q"], d["k_cache"], d["v_cache"], d["block_tables"], d["context_lens"],
                  wl.scale, max_context_len=batch.max_context_len, workspace=ws)
    return out


@pytest.fixture(params=["auto", "pp", "mma"])
def prefix_kernel(request, monkeypatch):
    """The shared-prefix pass through the default kernel (tcgen05 over 64-key
    tiles at head_dim 128), the tcgen05 ping-pong kernel over 128-key tiles
    and the mma.sync cluster kernel."""
    if request.param == "auto":
        monkeypatch.delenv("PA_PREFIX_KERNEL", raising=False)
    else:
        monkeypatch.setenv("PA_PREFIX_KERNEL", request.param)
    return request.param


def _run(lib, wl, rows=None):
    vals = workloads.values(wl)
    batch = build_batch(wl)
    d = device_inputs(wl, vals, batch)
    _prepare(lib, wl, batch, d)
    gs, gb, mg = _groups(batch, wl.block_size)
    assert int(gb.max()) > 0, "the workload must share blocks"
    out = _shared(lib, wl, batch, d, gs, gb, mg)
    torch.cuda.synchronize()
    assert lib.pa_get_device_error() == 0
    _, _, ref = oracle_step(wl, vals, rows=rows)
    assert_close(out, ref, wl.dtype, rows=rows, what=wl.name + " shared-prefix")
    return wl, batch, d, out


@pytest.mark.parametrize("cfg", ["4s", "4cows"])
def test_small_configs(lib, prefix_kernel, cfg):
    _run(lib, workloads.make(cfg))


@pytest.mark.parametrize("cfg", ["4", "4cow"])
def test_full_configs(lib, cfg):
    """Full-size parallel-sampling batches, every row."""
    _run(lib, workloads.make(cfg))


def test_agrees_with_plain_decode(lib):
    wl, batch, d, out = _run(lib, workloads.make("4s"))
    plain = _plain(lib, wl, batch, d).float()
    # two bf16 roundings of nearly equal fp32 values differ by at most 1 ulp
    # of the larger one (2^-7 of it covers an ulp in any binade)
    diff = (out.float() - plain).abs()
    assert torch.all(diff <= 2.0 ** -7 * torch.maximum(out.float().abs(), plain.abs()) + 1e-6), diff.max()


@pytest.mark.parametrize("H,Hk,D,bs,dtype,samples", [
    (32, 8, 128, 16, "bf16", 8),    # group 4: 16 members per prefix tile
    (16, 2, 64, 32, "f16", 8),      # group 8, head_dim 64, block 32
    (32, 2, 128, 16, "bf16", 8),    # group 16: 4 members per tile -> 2 member chunks
    (8, 8, 64, 16, "bf16", 5),      # group 1 (MHA)
    (64, 8, 128, 32, "bf16", 11),   # 11 samples of group 8 -> chunks of 8 and 3
    (24, 8, 128, 16, "f16", 7),     # group 3: 21 members per tile, 63 rows
])
def test_shapes(lib, prefix_kernel, H, Hk, D, bs, dtype, samples):
    wl = workloads.shared_prefix_workload(f"sp_{H}_{Hk}_{D}_{bs}_{dtype}_{samples}", 4100 + H + bs,
                                          3, samples, 5 * bs + 3, 3 * bs, H, Hk, D, bs, dtype)
    _run(lib, wl)


@pytest.mark.parametrize("cluster", ["1", "2", "8"])
def test_cluster_sizes(lib, monkeypatch, cluster):
    monkeypatch.setenv("PA_PREFIX_CLUSTER", cluster)
    _run(lib, workloads.make("4s"))


def _setup(lib, cfg="4s"):
    wl = workloads.make(cfg)
    vals = workloads.values(wl)
    batch = build_batch(wl)
    d = device_inputs(wl, vals, batch)
    _prepare(lib, wl, batch, d)
    torch.cuda.synchronize()
    kp = workloads.to_numpy_raw(d["k_cache"].cpu())
    vp = workloads.to_numpy_raw(d["v_cache"].cpu())
    qn = workloads.to_numpy_raw(vals["q"])
    return wl, batch, d, kp, vp, qn


def _ref(wl, qn, kp, vp, bt, cl):
    return oracle.decode(qn, kp, vp, np.asarray(bt, dtype=np.int32), np.asarray(cl, dtype=np.int32),
                         wl.scale, wl.dtype)


def test_member_with_only_shared_keys(lib, prefix_kernel):
    wl, batch, d, kp, vp, qn = _setup(lib)
    gs, gb, mg = _groups(batch, wl.block_size)
    p = int(gb[0])
    cl = batch.context_lens.copy()
    cl[3] = p * wl.block_size       # every key of sequence 3 is in the shared prefix
    cl[0] = p * wl.block_size + 1   # the group's first sequence: one private key
    out = _shared(lib, wl, batch, d, gs, gb, mg, context_lens=torch.from_numpy(cl).cuda())
    assert lib.pa_get_device_error() == 0
    assert_close(out, _ref(wl, qn, kp, vp, batch.block_tables, cl), wl.dtype, what="shared-only member")


def test_groups_not_covering_the_batch(lib):
    wl, batch, d, kp, vp, qn = _setup(lib)
    p = int(shared_prefix_groups(batch.block_tables, batch.context_lens, wl.block_size)[1][0])
    # sequences 0..1 and 6..15 are plain decode; 2..5 one group sharing p-2 blocks
    gs = torch.tensor([2, 6], dtype=torch.int32, device="cuda")
    gb = torch.tensor([p - 2], dtype=torch.int32, device="cuda")
    out = _shared(lib, wl, batch, d, gs, gb, 4)
    assert lib.pa_get_device_error() == 0
    assert_close(out, _ref(wl, qn, kp, vp, batch.block_tables, batch.context_lens), wl.dtype,
                 what="partial cover")


def test_no_groups_is_plain_decode(lib):
    wl, batch, d, kp, vp, qn = _setup(lib)
    gs = torch.zeros(1, dtype=torch.int32, device="cuda")
    gb = torch.zeros(0, dtype=torch.int32, device="cuda")
    out = _shared(lib, wl, batch, d, gs, gb, 1)
    assert lib.pa_get_device_error() == 0
    assert_close(out, _ref(wl, qn, kp, vp, batch.block_tables, batch.context_lens), wl.dtype,
                 what="no groups")


def test_member_table_mismatch(lib, prefix_kernel):
    wl, batch, d, kp, vp, qn = _setup(lib)
    gs, gb, mg = _groups(batch, wl.block_size)
    bt = batch.block_tables.copy()
    bt[2, 1] = bt[9, 1]              # sequence 2 no longer holds its group's block 1
    out = _shared(lib, wl, batch, d, gs, gb, mg, block_tables=torch.from_numpy(bt).cuda())
    assert lib.pa_get_device_error() & lib.PA_DEVERR_PREFIX
    assert torch.count_nonzero(out[2]) == 0
    keep = [i for i in range(batch.num_seqs) if i != 2]
    ref = _ref(wl, qn, kp, vp, bt, batch.context_lens)
    assert_close(out, ref, wl.dtype, rows=keep, what="other members")


def test_context_shorter_than_prefix(lib, prefix_kernel):
    wl, batch, d, kp, vp, qn = _setup(lib)
    gs, gb, mg = _groups(batch, wl.block_size)
    cl = batch.context_lens.copy()
    cl[5] = int(gb[0]) * wl.block_size - 3
    out = _shared(lib, wl, batch, d, gs, gb, mg, context_lens=torch.from_numpy(cl).cuda())
    assert lib.pa_get_device_error() & lib.PA_DEVERR_PREFIX
    assert torch.count_nonzero(out[5]) == 0
    keep = [i for i in range(batch.num_seqs) if i != 5]
    assert_close(out, _ref(wl, qn, kp, vp, batch.block_tables, cl), wl.dtype, rows=keep,
                 what="other members")


def test_bad_block_id_in_shared_range(lib, prefix_kernel):
    wl, batch, d, kp, vp, qn = _setup(lib)
    gs, gb, mg = _groups(batch, wl.block_size)
    bt = batch.block_tables.copy()
    bt[8:16, 2] = 1 << 30            # the second group's block 2, in every member's table
    out = _shared(lib, wl, batch, d, gs, gb, mg, block_tables=torch.from_numpy(bt).cuda())
    assert lib.pa_get_device_error() & lib.PA_DEVERR_BLOCK_ID
    assert torch.count_nonzero(out[8:16]) == 0
    assert_close(out, _ref(wl, qn, kp, vp, batch.block_tables, batch.context_lens), wl.dtype,
                 rows=range(8), what="first group")


def test_malformed_groups_fall_back_to_full_decode(lib):
    wl, batch, d, kp, vp, qn = _setup(lib)
    gs, gb, mg = _groups(batch, wl.block_size)
    bad = torch.tensor([0, 10, 8, 16], dtype=torch.int32, device="cuda")  # decreasing boundary
    gb3 = torch.tensor([int(gb[0])] * 3, dtype=torch.int32, device="cuda")
    out = _shared(lib, wl, batch, d, bad, gb3, 10)
    assert lib.pa_get_device_error() & lib.PA_DEVERR_PREFIX
    assert_close(out, _ref(wl, qn, kp, vp, batch.block_tables, batch.context_lens), wl.dtype,
                 what="malformed groups")


def test_host_argument_errors(lib):
    wl, batch, d, kp, vp, qn = _setup(lib)
    gs, gb, mg = _groups(batch, wl.block_size)
    with pytest.raises(lib.PAError) as e:   # no workspace
        lib.pa_decode_shared_prefix(torch.empty_like(d["q"]), d["q"], d["k_cache"], d["v_cache"],
                                    d["block_tables"], d["context_lens"], gs, gb, wl.scale)
    assert e.value.status == -3
    with pytest.raises(lib.PAError) as e:   # fp32 caches have no shared-prefix kernel
        q32 = d["q"].float()
        lib.pa_decode_shared_prefix(torch.empty_like(q32), q32, d["k_cache"].float(),
                                    d["v_cache"].float(), d["block_tables"], d["context_lens"],
                                    gs, gb, wl.scale)
    assert e.value.status == -2
    raw = lib.library()
    rc = raw.pa_decode_shared_prefix(d["q"].data_ptr(), d["q"].data_ptr() + 16, d["k_cache"].data_ptr(),
                                     d["v_cache"].data_ptr(), d["block_tables"].data_ptr(),
                                     batch.max_blocks_per_seq, d["context_lens"].data_ptr(),
                                     batch.num_seqs, None, None, 2, 8, wl.num_heads, wl.num_kv_heads,
                                     wl.head_dim, wl.block_size, wl.num_blocks, 0.1, 0, 2, None, 0,
                                     None)
    assert rc == -1  # group arrays missing
