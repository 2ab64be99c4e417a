"""pa_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers cannot hand the library a workspace: a plugin whose host
framework owns every byte of device memory, a runtime whose memory budget is
fixed at start-up, or a serving loop that must not call cudaMalloc on its hot
path.  pa_decode_noalloc runs pa_decode's kernels on a scratch array built
into the library instead.  Checked through the C ABI, on two calls in a row,
against the CPU oracle at the decode tolerance of the other GPU tests and
against pa_decode (with a workspace) bit for bit -- both run the same kernels
on the same partition.  Before the target batch, a different batch goes
through the same scratch, so stale partial records of another geometry are in
the array when the target batch starts.  This file is collected last so that
a run stopping at its first failure has already run everything else.
"""
import numpy as np
import pytest
import torch

import workloads
from gpu_harness import TOL, oracle_step
from paged_kv_cache_388_b200.batch import build_batch

pytestmark = pytest.mark.gpu


def _make(cfg):
    if cfg == "g16":  # 32 query heads on 2 KV heads (group 16), head_dim 128
        return workloads.decode_workload("noalloc_g16", 3900, [1, 17, 300, 900, 2048, 4000],
                                         32, 2, 128, 16, "bf16")
    return workloads.make(cfg)


def _inputs(wl):
    vals = workloads.values(wl)
    b = build_batch(wl)
    d = {k: vals[k].cuda() for k in ("q", "k_pool", "v_pool", "new_key", "new_value")}
    d["bt"] = torch.from_numpy(b.block_tables).cuda()
    d["cl"] = torch.from_numpy(b.context_lens).cuda()
    d["slots"] = torch.from_numpy(b.slot_mapping).cuda()
    return vals, b, d


def _noalloc(lib, wl, b, d, split):
    out = torch.full_like(d["q"], float("nan"))
    lib.pa_decode_noalloc(out, d["q"], d["k_pool"], d["v_pool"], d["bt"], d["cl"], wl.scale,
                          max_context_len=b.max_context_len, kv_split_tokens=split)
    torch.cuda.synchronize()
    assert lib.pa_get_device_error() == 0
    return out


@pytest.mark.parametrize("cfg,split,stale_cfg,stale_split",
                         [("3s", 0, "4s", 64), ("3s32", 0, "3s", 64), ("4s", 64, "3s32", 0),
                          ("g16", 0, "3s", 0)])
def test_noalloc_matches_oracle_and_pa_decode_twice(cfg, split, stale_cfg, stale_split):
    from paged_kv_cache_388_b200 import _lib
    # another batch first: its partials are left in the shared scratch
    swl = _make(stale_cfg)
    _, sb, sd = _inputs(swl)
    _noalloc(_lib, swl, sb, sd, stale_split)

    wl = _make(cfg)
    vals, b, d = _inputs(wl)
    _lib.pa_reshape_and_cache(d["new_key"], d["new_value"], d["k_pool"], d["v_pool"], d["slots"])
    ws = torch.empty(max(16, _lib.pa_decode_workspace_size(
        b.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.block_size,
        b.max_context_len, split)), dtype=torch.uint8, device="cuda")
    ref = torch.empty_like(d["q"])
    _lib.pa_decode(ref, d["q"], d["k_pool"], d["v_pool"], d["bt"], d["cl"], wl.scale,
                   max_context_len=b.max_context_len, kv_split_tokens=split, workspace=ws)
    _, _, oracle_out = oracle_step(wl, vals)
    atol, rtol = TOL[wl.dtype]
    for _ in range(2):
        out = _noalloc(_lib, wl, b, d, split)
        assert torch.equal(out, ref), "noalloc differs from pa_decode on the same kernels"
        g = out.float().cpu().numpy().astype(np.float64)
        assert np.all(np.abs(g - oracle_out) <= atol + rtol * np.abs(oracle_out))


def test_noalloc_rejects_batches_beyond_its_scratch():
    from paged_kv_cache_388_b200 import _lib
    wl = workloads.make("3s")
    _, b, d = _inputs(wl)
    cap = _lib.pa_noalloc_scratch_bytes()
    # forced 16-token splits over a long max context: more partials than fit
    split, max_ctx = 16, 1 << 20
    need = _lib.pa_decode_workspace_size(b.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim,
                                         wl.block_size, max_ctx, split)
    assert need > cap
    bt = torch.zeros(b.num_seqs, max_ctx // wl.block_size, dtype=torch.int32, device="cuda")
    bt[:, : d["bt"].shape[1]] = d["bt"]
    out = torch.zeros_like(d["q"])
    with pytest.raises(_lib.PAError) as e:
        _lib.pa_decode_noalloc(out, d["q"], d["k_pool"], d["v_pool"], bt, d["cl"], wl.scale,
                               max_context_len=max_ctx, kv_split_tokens=split)
    assert e.value.status == -3
    assert torch.count_nonzero(out) == 0  # nothing was launched
