"""Shared helpers for the GPU parity tests: run one step of the hot path on the
device (copy_blocks -> reshape_and_cache -> decode) and the same step in the
CPU oracle, on the same seeded inputs."""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import oracle
import workloads
from model_batch import model_batch

TOL = {"f32": (1e-5, 1e-5), "f16": (2e-3, 1e-2), "bf16": (2e-3, 1e-2)}


def device_inputs(wl, vals, batch, device="cuda"):
    d = {
        "q": vals["q"].to(device),
        "k_cache": vals["k_pool"].to(device),
        "v_cache": vals["v_pool"].to(device),
        "key": vals["new_key"].to(device),
        "value": vals["new_value"].to(device),
        "block_tables": torch.from_numpy(batch.block_tables).to(device),
        "context_lens": torch.from_numpy(batch.context_lens).to(device),
        "slot_mapping": torch.from_numpy(batch.slot_mapping).to(device),
        "cow": torch.from_numpy(np.ascontiguousarray(batch.cow_pairs)).to(device),
        "qsl": None if batch.query_start_loc is None else torch.from_numpy(batch.query_start_loc).to(device),
    }
    return d


def gpu_step(lib, wl, batch, d, kv_split_tokens=0):
    """The hot path through the C ABI: returns out [Tq, H, D] on the device."""
    if d["cow"].shape[0]:
        lib.pa_copy_blocks(d["k_cache"], d["v_cache"], d["cow"])
    lib.pa_reshape_and_cache(d["key"], d["value"], d["k_cache"], d["v_cache"], d["slot_mapping"])
    out = torch.empty_like(d["q"])
    ws_bytes = lib.pa_decode_workspace_size(batch.num_seqs, wl.num_heads, wl.num_kv_heads,
                                            wl.head_dim, wl.block_size, batch.max_context_len,
                                            kv_split_tokens)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=d["q"].device)
    lib.pa_decode(out, d["q"], d["k_cache"], d["v_cache"], d["block_tables"], d["context_lens"],
                  wl.scale, query_start_loc=d["qsl"], max_query_len=batch.max_query_len,
                  max_context_len=batch.max_context_len, kv_split_tokens=kv_split_tokens,
                  workspace=ws)
    return out


def oracle_step(wl, vals, rows=None):
    """The same step in the oracle, from the oracle's own allocation model."""
    mb = model_batch(wl)
    kp = workloads.to_numpy_raw(vals["k_pool"]).copy()
    vp = workloads.to_numpy_raw(vals["v_pool"]).copy()
    if mb["cow_pairs"].shape[0]:
        oracle.copy_blocks(kp, vp, mb["cow_pairs"], wl.dtype)
    oracle.reshape_and_cache(kp, vp, workloads.to_numpy_raw(vals["new_key"]),
                             workloads.to_numpy_raw(vals["new_value"]), mb["slot_mapping"], wl.dtype)
    out = oracle.decode(workloads.to_numpy_raw(vals["q"]), kp, vp, mb["block_tables"],
                        mb["context_lens"], wl.scale, wl.dtype,
                        query_start_loc=mb["query_start_loc"], rows=rows)
    return kp, vp, out


def raw_cpu(t):
    return workloads.to_numpy_raw(t.cpu())


def _log_errors(what, dtype, rows_checked, max_abs, max_rel):
    """Append the comparison's error figures to $PA_PARITY_LOG (JSON lines)
    when that variable is set, and print them (visible with pytest -s)."""
    rec = {"what": what, "dtype": dtype, "rows_checked": rows_checked, "max_abs": max_abs,
           "max_rel_ref_gt_1e-3": max_rel}
    print("parity", json.dumps(rec))
    path = os.environ.get("PA_PARITY_LOG")
    if path:
        with open(path, "a", encoding="utf-8") as f:
            f.write(json.dumps(rec) + "\n")


def assert_close(got, want, dtype, rows=None, what=""):
    """Element-wise |got - want| <= atol + rtol*|want| at the dtype's
    tolerance; returns the max absolute error and logs it together with the
    max relative error over elements with |want| > 1e-3."""
    atol, rtol = TOL[dtype]
    g = got.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        rows = np.asarray(sorted(rows))
        g, want = g[rows], want[rows]
    err = np.abs(g - want)
    bound = atol + rtol * np.abs(want)
    bad = err > bound
    big = np.abs(want) > 1e-3
    max_rel = float((err[big] / np.abs(want[big])).max()) if big.any() else 0.0
    _log_errors(what, dtype, int(g.shape[0]), float(err.max()) if err.size else 0.0, max_rel)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} elements outside |d| <= {atol} + {rtol}|ref|; "
            f"max abs {err.max():.3g}; first bad {idx.tolist()} got {g[bad][:5]} want {want[bad][:5]}")
    return float(err.max()) if err.size else 0.0
