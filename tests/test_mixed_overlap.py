"""A mixed batch's chunk rows run on a side stream beside its decode rows.

pa_decode forks the chunk-row kernel of a batch that mixes chunked-prefill
rows with decode rows onto a stream of the device's highest priority and
joins it back into the caller's stream with events, so that the tensor-bound
chunk rows and the HBM-bound decode rows share the SMs.  pa_decode_noalloc
keeps both on the caller's stream, one after the other.  The two run the same
kernels on disjoint output rows, so their outputs agree bit for bit, and both
agree with the oracle.  The join must order later work on the caller's
stream after the chunk rows, also inside a CUDA graph capture.
"""
import numpy as np
import pytest
import torch

import workloads
from gpu_harness import assert_close, device_inputs, oracle_step
from paged_kv_cache_388_b200.batch import build_batch

pytestmark = pytest.mark.gpu


def _setup(cfg):
    from paged_kv_cache_388_b200 import _lib
    wl = workloads.make(cfg) if isinstance(cfg, str) else cfg
    vals = workloads.values(wl)
    batch = build_batch(wl)
    d = device_inputs(wl, vals, batch)
    _lib.pa_reshape_and_cache(d["key"], d["value"], d["k_cache"], d["v_cache"], d["slot_mapping"])
    ws = torch.empty(max(16, _lib.pa_decode_workspace_size(
        batch.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.block_size,
        batch.max_context_len, 0)), dtype=torch.uint8, device="cuda")
    return _lib, wl, vals, batch, d, ws


def _forked(lib, wl, batch, d, ws, out):
    lib.pa_decode(out, d["q"], d["k_cache"], d["v_cache"], d["block_tables"], d["context_lens"],
                  wl.scale, query_start_loc=d["qsl"], max_query_len=batch.max_query_len,
                  max_context_len=batch.max_context_len, workspace=ws)


@pytest.mark.parametrize("cfg", ["5s", "5s32"])
def test_forked_matches_serial_and_oracle(cfg):
    lib, wl, vals, batch, d, ws = _setup(cfg)
    assert batch.max_query_len > 1 and int(batch.context_lens.shape[0]) > 2
    out = torch.full_like(d["q"], float("nan"))
    _forked(lib, wl, batch, d, ws, out)
    # stream order: a copy enqueued right after the call sees every row
    seen = out.clone()
    serial = torch.full_like(d["q"], float("nan"))
    lib.pa_decode_noalloc(serial, d["q"], d["k_cache"], d["v_cache"], d["block_tables"],
                          d["context_lens"], wl.scale, query_start_loc=d["qsl"],
                          max_query_len=batch.max_query_len, max_context_len=batch.max_context_len)
    torch.cuda.synchronize()
    assert lib.pa_get_device_error() == 0
    assert torch.equal(out, serial), "side-stream chunk rows differ from the serial order"
    assert torch.equal(seen, out), "work after the call ran before the chunk rows finished"
    _, _, ref = oracle_step(wl, vals)
    assert_close(out, ref, wl.dtype, what=f"{wl.name} forked")


def test_forked_call_in_cuda_graph():
    """Captured and replayed: the fork and join become graph edges, and a
    kernel captured after the call reads the finished chunk rows."""
    lib, wl, vals, batch, d, ws = _setup("5s")
    eager = torch.empty_like(d["q"])
    _forked(lib, wl, batch, d, ws, eager)  # first call outside the capture
    torch.cuda.synchronize()
    out = torch.empty_like(d["q"])
    after = torch.empty_like(d["q"])
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _forked(lib, wl, batch, d, ws, out)
        after.copy_(out * 1)
    for _ in range(3):
        out.fill_(float("nan"))
        after.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert lib.pa_get_device_error() == 0
        assert torch.equal(out, eager)
        assert torch.equal(after, eager)
    del g


def test_forked_mixed_8k_long_chunks():
    """Config 5's chunk shape at half the prefix, with decode rows long enough
    that their CTAs outlive the first wave of chunk CTAs: every row against the
    oracle, and bit for bit against the serial order."""
    wl = workloads.mixed_workload("overlap_mixed_8k", 4343, 4, 30000, 60000, 4, 8192, 512, 32, 8,
                                  128, 16, "bf16")
    lib, wl, vals, batch, d, ws = _setup(wl)
    out = torch.empty_like(d["q"])
    _forked(lib, wl, batch, d, ws, out)
    serial = torch.empty_like(d["q"])
    lib.pa_decode_noalloc(serial, d["q"], d["k_cache"], d["v_cache"], d["block_tables"],
                          d["context_lens"], wl.scale, query_start_loc=d["qsl"],
                          max_query_len=batch.max_query_len, max_context_len=batch.max_context_len)
    torch.cuda.synchronize()
    assert lib.pa_get_device_error() == 0
    assert torch.equal(out, serial)
    qsl = batch.query_start_loc
    rows = [int(qsl[i]) for i in range(len(qsl) - 1) if qsl[i + 1] - qsl[i] == 1]
    rows += list(range(int(qsl[-1]) - 64, int(qsl[-1])))  # the last chunk's final rows
    _, _, ref = oracle_step(wl, vals, rows=np.asarray(rows))
    assert_close(out, ref, wl.dtype, rows=rows, what="overlap_mixed_8k")


def test_concurrent_callers():
    """Two host threads, each with its own stream and workspace, call
    pa_decode on mixed batches at once: the library's side stream is shared,
    so each fork-join holds it; every result equals the serial order's."""
    import threading
    lib, wl, vals, batch, d, _ = _setup("5s")
    serial = torch.empty_like(d["q"])
    lib.pa_decode_noalloc(serial, d["q"], d["k_cache"], d["v_cache"], d["block_tables"],
                          d["context_lens"], wl.scale, query_start_loc=d["qsl"],
                          max_query_len=batch.max_query_len, max_context_len=batch.max_context_len)
    torch.cuda.synchronize()
    size = lib.pa_decode_workspace_size(batch.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim,
                                        wl.block_size, batch.max_context_len, 0)
    outs, errors = [], []

    def worker():
        try:
            st = torch.cuda.Stream()
            ws = torch.empty(max(16, size), dtype=torch.uint8, device="cuda")
            res = [torch.empty_like(d["q"]) for _ in range(6)]
            with torch.cuda.stream(st):
                for o in res:
                    _forked(lib, wl, batch, d, ws, o)
            st.synchronize()
            outs.extend(res)
        except Exception as e:  # noqa: BLE001 -- surfaced below
            errors.append(e)

    threads = [threading.Thread(target=worker) for _ in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    assert lib.pa_get_device_error() == 0
    assert len(outs) == 12
    for o in outs:
        assert torch.equal(o, serial)
