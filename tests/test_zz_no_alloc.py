"""pa_decode_noalloc: decode for callers that cannot allocate device memory.

It runs pa_decode's kernels on a scratch array built into the library instead
of a caller workspace.  Checked through the C ABI against pa_decode (with a
workspace) on the same inputs, on two calls in a row (the second one reuses
the scratch the first one left behind), within the decode tolerance of the
other GPU tests.  This file is collected last so that a run stopping at its
first failure has already run everything else.
"""
import numpy as np
import pytest
import torch

import workloads
from paged_kv_cache_388_b200.batch import build_batch

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-3, 1e-2  # bf16 decode tolerance used by the parity tests


def _inputs(cfg):
    wl = workloads.make(cfg)
    vals = workloads.values(wl)
    b = build_batch(wl)
    d = {k: vals[k].cuda() for k in ("q", "k_pool", "v_pool", "new_key", "new_value")}
    d["bt"] = torch.from_numpy(b.block_tables).cuda()
    d["cl"] = torch.from_numpy(b.context_lens).cuda()
    d["slots"] = torch.from_numpy(b.slot_mapping).cuda()
    return wl, b, d


@pytest.mark.parametrize("cfg,split", [("3s", 0), ("3s32", 0), ("4s", 64)])
def test_noalloc_matches_pa_decode_twice(cfg, split):
    from paged_kv_cache_388_b200 import _lib
    wl, b, d = _inputs(cfg)
    _lib.pa_reshape_and_cache(d["new_key"], d["new_value"], d["k_pool"], d["v_pool"], d["slots"])
    ws = torch.empty(max(16, _lib.pa_decode_workspace_size(
        b.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.block_size,
        b.max_context_len, split)), dtype=torch.uint8, device="cuda")
    ref = torch.empty_like(d["q"])
    _lib.pa_decode(ref, d["q"], d["k_pool"], d["v_pool"], d["bt"], d["cl"], wl.scale,
                   max_context_len=b.max_context_len, kv_split_tokens=split, workspace=ws)
    for _ in range(2):
        out = torch.full_like(d["q"], float("nan"))
        _lib.pa_decode_noalloc(out, d["q"], d["k_pool"], d["v_pool"], d["bt"], d["cl"], wl.scale,
                               max_context_len=b.max_context_len, kv_split_tokens=split)
        torch.cuda.synchronize()
        assert _lib.pa_get_device_error() == 0
        g, r = out.float().cpu().numpy(), ref.float().cpu().numpy()
        assert np.all(np.abs(g - r) <= ATOL + RTOL * np.abs(r))


def test_noalloc_rejects_batches_beyond_its_scratch():
    from paged_kv_cache_388_b200 import _lib
    wl, b, d = _inputs("3s")
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
