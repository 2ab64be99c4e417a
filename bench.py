#!/usr/bin/env python
"""Benchmark: one decode step of paged attention on the Llama-3-8B-shaped GQA batch,
then every other workload of the build measured call by call.

Headline (the JSON line's ``value``): a step is the whole hot path over one
batch -- copy-on-write block copies (none in this batch), reshape_and_cache of
the step's 256 new tokens, then paged decode attention of the 256 query tokens
over their block-table KV cache (32 query heads / 8 KV heads, head_dim 128,
block size 16, bf16, context lengths lognormal with median 800 capped at 4096,
shuffled pool); achieved HBM GB/s of the step (algorithmic bytes / device
time) and decode tokens/s.

``configs`` (N = 1): every workload -- Llama-2-7B-shaped MHA fp16, the
Llama-3-8B-shaped batch in bf16 and with an FP8 (E4M3) cache, the
parallel-sampling shared-prefix batch (shared-prefix call and plain decode,
also with copy-on-write), the long-context batch with chunked-prefill rows at
block size 16 and 32 (whole call, decode rows alone, chunk rows alone), the
tiny fp32 batch -- each call timed as the median (min, max) of 50 calls with
the L2 flushed before every one, against its roofline (HBM copy bandwidth for
decode, the bf16 tensor peak for chunk rows, the larger of the two bounds for
a mixed call).

``cpu_baseline``: the CPU oracle (fp64) on the machine's host cores on bounded
samples: the headline step, and per workload a sample of query rows timed
with all threads (and one thread for the first three workloads), with the
largest absolute and relative differences between those rows and the GPU's.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 is launched with torchrun: every rank runs its own batch (weak scaling,
no collective on the data path); times are the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import gc
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402
from paged_kv_cache_388_b200.batch import (build_batch, shared_prefix_groups,  # noqa: E402
                                           staged_blocks_needed)

METRIC = "paged decode attention: achieved HBM GB/s (% of peak) and decode tokens/s"
UNIT = "GB/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_TFLOPS = 1590.0
L2_BYTES = 126 * 2 ** 20
FLUSH_BYTES = 256 * 2 ** 20          # >= 2x L2: reading this evicts every cached line
EXTRA_CONFIGS = ("2", "3fp8", "4", "4cow", "4fp8", "5", "5bs32", "5fp8", "1")


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f)
    return None


def hbm_peak():
    pk = _peaks()
    if pk and "hbm_gbs" in pk:
        return float(pk["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    pk = _peaks()
    if pk and "bf16_tflops" in pk:
        return float(pk["bf16_tflops"]), "measured"
    return FALLBACK_TFLOPS, "fallback"


KERNEL_SOURCES = ("paged_kv_cache_388_b200/csrc/decode_mma.cu",
                  "paged_kv_cache_388_b200/csrc/decode_common.cuh",
                  "paged_kv_cache_388_b200/csrc/pa_device.cuh",
                  "paged_kv_cache_388_b200/csrc/pa_internal.h")
PROFILE = os.path.join(ROOT, "profiles", "paged_decode_mma_kernel_cfg3.md")


def profiled_traffic(config):
    """DRAM bytes per launch of the decode kernel from the committed ncu
    summary, or None if that summary is for other sources or another workload."""
    import hashlib
    if config != "3" or not os.path.exists(PROFILE):
        return None
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    fields = {}
    with open(PROFILE, encoding="utf-8") as fh:
        for line in fh:
            if ":" in line and line.split(":")[0] in ("traffic_bytes_per_launch", "source_sha256"):
                k, val = line.split(":", 1)
                fields[k.strip()] = val.strip()
    if fields.get("source_sha256") != h.hexdigest():
        return None
    return int(fields["traffic_bytes_per_launch"])


def chunk_flops(batch, seqs=None):
    """Multiply-add FLOPs of the chunked-query rows (QK^T and PV over the keys
    each row may see), per head and head_dim unit: sum over rows of visible
    keys (multiply by H * D * 4 for FLOPs)."""
    qsl = batch.query_start_loc
    if qsl is None:
        return 0
    total = 0
    for i, L in enumerate(batch.context_lens.tolist()):
        if seqs is not None and i not in seqs:
            continue
        Q = int(qsl[i + 1] - qsl[i])
        if Q <= 1:
            continue
        total += sum(L - Q + t + 1 for t in range(Q))
    return total


def sub_batch(batch, keep):
    """Rows of the batch for the sequences `keep` (decode-only or chunk-only)."""
    keep = list(keep)
    bt = batch.block_tables[keep]
    cl = batch.context_lens[keep]
    qsl = batch.query_start_loc
    if qsl is None:
        return bt, cl, None, np.asarray(keep, dtype=np.int64)
    rows, starts = [], [0]
    for i in keep:
        rows.extend(range(int(qsl[i]), int(qsl[i + 1])))
        starts.append(len(rows))
    return bt, cl, np.asarray(starts, dtype=np.int32), np.asarray(rows, dtype=np.int64)


def elem_bytes(dtype):
    return {"f32": 4, "f16": 2, "bf16": 2}[dtype]


def seq_bytes(wl, batch, seqs, kv_elem=None):
    """Algorithmic bytes of the step restricted to sequences `seqs`: every
    byte the method has to move, once (shared physical blocks once).
    kv_elem: bytes per cached element when it differs from q's (FP8 cache)."""
    e = elem_bytes(wl.dtype)
    ekv = e if kv_elem is None else kv_elem
    H, Hk, D, bs = wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.block_size
    seen = set()
    kv_tokens = 0
    nblk_total = 0
    qrows = 0
    for i in seqs:
        L = int(batch.context_lens[i])
        nblk = -(-L // bs)
        nblk_total += nblk
        for j in range(nblk):
            pb = int(batch.block_tables[i, j])
            if pb not in seen:
                seen.add(pb)
                kv_tokens += min(bs, L - j * bs)
        qsl = batch.query_start_loc
        qrows += 1 if qsl is None else int(qsl[i + 1] - qsl[i])
    decode = kv_tokens * 2 * Hk * D * ekv + 2 * qrows * H * D * e + nblk_total * 4 + len(seqs) * 4
    return decode, kv_tokens, qrows


def step_bytes(wl, batch, kv_elem=None):
    e = elem_bytes(wl.dtype)
    ekv = e if kv_elem is None else kv_elem
    Hk, D, bs = wl.num_kv_heads, wl.head_dim, wl.block_size
    decode, kv_tokens, qrows = seq_bytes(wl, batch, range(batch.num_seqs), kv_elem)
    t_new = wl.num_new_tokens
    reshape = 2 * (t_new * Hk * D * (e + ekv)) + t_new * 8
    copy = int(batch.cow_pairs.shape[0]) * 2 * (2 * Hk * bs * D * ekv)
    return {"decode": decode, "reshape": reshape, "copy_blocks": copy,
            "step": decode + reshape + copy, "kv_tokens": kv_tokens, "q_rows": qrows}


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.fh = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        self.fh = os.fdopen(fd, "w")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.fh.close()

    def summary(self):
        sm, smax, reasons = [], [], set()
        try:
            with open(self.path) as f:
                lines = f.readlines()
            os.unlink(self.path)
        except OSError:
            lines = []
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(self.NAMES, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "samples": len(sm),
                "reasons": sorted(reasons)}


def aggregate(local_bytes, local_ms, device):
    """Whole-job totals over ranks: bytes summed, time = the slowest rank's.
    No-op without an initialised process group."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(local_bytes), float(local_ms)
    b = torch.tensor([float(local_bytes)], dtype=torch.float64, device=device)
    t = torch.tensor([float(local_ms)], dtype=torch.float64, device=device)
    dist.all_reduce(b, op=dist.ReduceOp.SUM)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(b.item()), float(t.item())


# --------------------------------------------------------------------------
# device timing
# --------------------------------------------------------------------------
class Timer:
    """CUDA-event timing on the launching stream.  Calls are captured into
    CUDA graphs so that host launch cost stays out of the device time."""

    def __init__(self, dev):
        self.dev = dev
        self.stream = torch.cuda.current_stream(dev)
        self._flush = None

    def _graph(self, fn, n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(n):
                fn()
        return g

    def back_to_back(self, fn, k):
        """Average ms of one call over k calls replayed back to back."""
        g = self._graph(fn, k)
        g.replay()
        torch.cuda.synchronize(self.dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(self.stream)
        g.replay()
        e1.record(self.stream)
        torch.cuda.synchronize(self.dev)
        del g
        return e0.elapsed_time(e1) / k

    def flushed(self, fn, warm=10, iters=50):
        """Median (min, max) ms of `iters` single calls, each preceded by a
        memset of FLUSH_BYTES that evicts the L2, after `warm` calls."""
        if self._flush is None:
            self._flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=self.dev)
        g = self._graph(fn, 1)
        for _ in range(warm):
            g.replay()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(iters)]
        torch.cuda.synchronize(self.dev)
        for e0, e1 in evs:
            # a read of FLUSH_BYTES evicts the L2 and leaves no dirty line to be
            # written back inside the timed call (~40 us; the replay is enqueued meanwhile)
            torch.amax(self._flush)
            e0.record(self.stream)
            g.replay()
            e1.record(self.stream)
        torch.cuda.synchronize(self.dev)
        ts = sorted(e0.elapsed_time(e1) for e0, e1 in evs)
        del g
        return {"median_ms": statistics.median(ts), "min_ms": ts[0], "max_ms": ts[-1],
                "calls": iters, "l2": "flushed before every call"}


# --------------------------------------------------------------------------
# one workload resident on the device
# --------------------------------------------------------------------------
def fp8_scale(*ts):
    return float(np.float32(max(float(t.float().abs().max()) for t in ts) / 448.0 * 1.25))


def fp8_quant(t, sc):
    return (t.float() / torch.tensor(sc, dtype=torch.float32)).to(torch.float8_e4m3fn).view(torch.uint8)


class DeviceBatch:
    """A workload's batch on the device with the calls of its step."""

    def __init__(self, cfg, dev, replica=0, kv_fp8=False, plain_decode=False):
        from paged_kv_cache_388_b200.session import PagedKVCache
        self.cfg = cfg
        self.wl = wl = workloads.make(cfg, replica=replica)
        self.batch = batch = build_batch(wl)
        self.vals = vals = workloads.values(wl)
        self.dev = dev
        self.kv_fp8 = kv_fp8
        if kv_fp8:
            # FP8 (E4M3) cache: one scale per tensor, the pool's history quantised
            # on the host, this step's K/V quantised by pa_reshape_and_cache_fp8
            self.ks = fp8_scale(vals["k_pool"], vals["new_key"])
            self.vs = fp8_scale(vals["v_pool"], vals["new_value"])
            self.k_codes = fp8_quant(vals["k_pool"], self.ks)
            self.v_codes = fp8_quant(vals["v_pool"], self.vs)
            self.cache = PagedKVCache(wl.num_blocks, wl.num_kv_heads, wl.head_dim, wl.block_size,
                                      dtype=torch.uint8, k_cache=self.k_codes.to(dev),
                                      v_cache=self.v_codes.to(dev), kv_scales=(self.ks, self.vs))
        else:
            self.cache = PagedKVCache(wl.num_blocks, wl.num_kv_heads, wl.head_dim, wl.block_size,
                                      k_cache=vals["k_pool"].to(dev), v_cache=vals["v_pool"].to(dev))
        self.q = vals["q"].to(dev)
        self.key = vals["new_key"].to(dev)
        self.value = vals["new_value"].to(dev)
        self.slot = torch.from_numpy(batch.slot_mapping).to(dev)
        self.bt = torch.from_numpy(batch.block_tables).to(dev)
        self.cl = torch.from_numpy(batch.context_lens).to(dev)
        self.qsl = None if batch.query_start_loc is None else torch.from_numpy(batch.query_start_loc).to(dev)
        self.cow = torch.from_numpy(np.ascontiguousarray(batch.cow_pairs)).to(dev)
        self.out = torch.empty_like(self.q)
        self.mcl = batch.max_context_len
        self.cache.workspace(batch.num_seqs, wl.num_heads, self.mcl)
        self.shared = wl.kind == "shared_prefix" and not plain_decode
        if self.shared:
            gs_np, gb_np = shared_prefix_groups(batch.block_tables, batch.context_lens, wl.block_size)
            self.gs = torch.from_numpy(gs_np).to(dev)
            self.gb = torch.from_numpy(gb_np).to(dev)
            self.gb_np = gb_np
            self.max_group = int(np.diff(gs_np).max())
        self.bytes = step_bytes(wl, batch, 1 if kv_fp8 else None)
        # an FP8 cache stages the blocks of chunk-row sequences: the bound is
        # counted here, on the host, not inside the timed (captured) calls
        self.staged = None
        if kv_fp8 and batch.query_start_loc is not None and batch.max_query_len > 1:
            self.staged = staged_blocks_needed(batch.query_start_loc, batch.context_lens,
                                               wl.block_size)

    def attend_plain(self):
        self.cache.attend(self.q, self.bt, self.cl, self.wl.scale, out=self.out,
                          query_start_loc=self.qsl, max_query_len=self.batch.max_query_len,
                          max_context_len=self.mcl, staged_blocks=self.staged)

    def attend(self):
        if self.shared:
            self.cache.attend_shared_prefix(self.q, self.bt, self.cl, self.gs, self.gb,
                                            self.wl.scale, max_group_size=self.max_group,
                                            out=self.out, max_context_len=self.mcl,
                                            staged_blocks=int(self.gb_np.sum()) if self.kv_fp8
                                            else None)
        else:
            self.attend_plain()

    def write(self):
        self.cache.write(self.key, self.value, self.slot)

    def copy_blocks(self):
        self.cache.copy_blocks(self.cow)

    def step(self):
        if self.cow.shape[0]:
            self.copy_blocks()
        self.write()
        self.attend()

    def launches_per_step(self):
        from paged_kv_cache_388_b200 import _lib
        b = self.batch
        splits = _lib.pa_decode_workspace_size(b.num_seqs, self.wl.num_heads, self.wl.num_kv_heads,
                                               self.wl.head_dim, self.wl.block_size, self.mcl, 0) > 0
        return 1 + 1 + (1 if splits else 0) + (1 if self.cow.shape[0] else 0) + \
            (1 if b.max_query_len > 1 else 0) + (1 if self.shared else 0) + \
            (2 if self.staged or (self.kv_fp8 and self.shared) else 0)  # FP8: staging plan + copy

    def rows_callable(self, ids):
        """A call attending only the query rows of sequences `ids` (the decode
        rows or the chunk rows of a mixed batch), into its own output."""
        sbt, scl, sqsl, srows = sub_batch(self.batch, ids)
        sq = self.q[torch.from_numpy(srows).to(self.dev)].contiguous()
        sout = torch.empty_like(sq)
        t_bt = torch.from_numpy(np.ascontiguousarray(sbt)).to(self.dev)
        t_cl = torch.from_numpy(np.ascontiguousarray(scl)).to(self.dev)
        t_qsl = None if sqsl is None else torch.from_numpy(sqsl).to(self.dev)
        mql = int(max(np.diff(sqsl))) if sqsl is not None else 1
        if t_qsl is not None and mql == 1:
            t_qsl = None
        mcl = int(scl.max())
        staged = None
        if self.kv_fp8 and t_qsl is not None:
            staged = staged_blocks_needed(sqsl, scl, self.wl.block_size)
        return lambda: self.cache.attend(sq, t_bt, t_cl, self.wl.scale, out=sout,
                                         query_start_loc=t_qsl, max_query_len=mql,
                                         max_context_len=mcl, staged_blocks=staged)


def _rate(nbytes, ms):
    return nbytes / (ms * 1e-3) / 1e9


def measure_config(db, timer, k):
    """Per-call timings of one workload against its rooflines."""
    wl, batch = db.wl, db.batch
    peak, peak_kind = hbm_peak()
    tc, tc_kind = tensor_peak()
    for _ in range(3):
        db.step()
    torch.cuda.synchronize(db.dev)
    res = {"workload": wl.name, "dtype": ("fp8_e4m3 KV, " + wl.dtype + " q/out") if db.kv_fp8
           else wl.dtype, "seqs": batch.num_seqs, "q_rows": db.bytes["q_rows"],
           "kv_tokens": db.bytes["kv_tokens"], "decode_bytes": db.bytes["decode"]}
    name = ("pa_decode_shared_prefix" if db.shared else "pa_decode") + ("_fp8" if db.kv_fp8 else "")
    call = timer.flushed(db.attend)
    call["avg_ms_back_to_back"] = timer.back_to_back(db.attend, k)
    call["GBps"] = _rate(db.bytes["decode"], call["median_ms"])
    call["frac_of_hbm_peak"] = call["GBps"] / peak
    call["tokens_per_s"] = db.bytes["q_rows"] / (call["median_ms"] * 1e-3)
    res[name] = call
    res["hbm_peak_GBps"] = {"value": peak, "kind": f"{peak_kind} copy bandwidth"}
    w = timer.flushed(db.write)
    w["GBps"] = _rate(db.bytes["reshape"], w["median_ms"])
    res["pa_reshape_and_cache_fp8" if db.kv_fp8 else "pa_reshape_and_cache"] = w
    if db.cow.shape[0]:
        c = timer.flushed(db.copy_blocks)
        c["pairs"] = int(db.cow.shape[0])
        c["GBps"] = _rate(db.bytes["copy_blocks"], c["median_ms"])
        res["pa_copy_blocks"] = c
    if db.shared:
        plain = timer.flushed(db.attend_plain)
        plain["GBps_unique"] = _rate(db.bytes["decode"], plain["median_ms"])
        res["pa_decode_plain"] = plain
        logical = int(batch.context_lens.astype(np.int64).sum()) * 2 * wl.num_kv_heads * \
            wl.head_dim * elem_bytes(wl.dtype)
        res[name]["logical_kv_bytes"] = logical
        res[name]["GBps_logical"] = _rate(logical, call["median_ms"])
        res[name]["groups"] = int(db.gb_np.shape[0])
        res[name]["shared_blocks"] = int(db.gb_np.max())
    if batch.query_start_loc is not None:
        qsl = batch.query_start_loc
        dec_ids = [i for i in range(batch.num_seqs) if qsl[i + 1] - qsl[i] == 1]
        chk_ids = [i for i in range(batch.num_seqs) if qsl[i + 1] - qsl[i] > 1]
        flops = chunk_flops(batch) * wl.num_heads * wl.head_dim * 4
        dbytes, _, _ = seq_bytes(wl, batch, dec_ids, kv_elem=1 if db.kv_fp8 else None)
        if dec_ids:
            d = timer.flushed(db.rows_callable(dec_ids))
            d["GBps"] = _rate(dbytes, d["median_ms"])
            d["frac_of_hbm_peak"] = d["GBps"] / peak
            d["bytes"] = dbytes
            res["decode_rows"] = d
        if chk_ids:
            c = timer.flushed(db.rows_callable(chk_ids))
            c["flops"] = flops
            c["TFLOPs"] = flops / (c["median_ms"] * 1e-3) / 1e12
            c["frac_of_tensor_peak"] = c["TFLOPs"] / tc
            res["chunk_rows"] = c
        bound_ms = max(db.bytes["decode"] / (peak * 1e9), flops / (tc * 1e12)) * 1e3
        res["mixed_bound"] = {"ms": bound_ms, "rule": "max(all bytes / HBM peak, chunk flops / "
                              "bf16 tensor peak)", "tensor_peak_TFLOPs": tc,
                              "tensor_peak_kind": tc_kind,
                              "frac": bound_ms / call["median_ms"]}
    # one whole step last, so that db.out is the step's output on the step's
    # cache (the lone copy_blocks / write timings above left other contents)
    db.step()
    torch.cuda.synchronize(db.dev)
    return res


# --------------------------------------------------------------------------
# CPU oracle legs (cpu_baseline and --impl reference)
# --------------------------------------------------------------------------
def host_cores():
    """Host cores this process may run on (its CPU affinity set)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_runner(wl, vals, batch):
    """Returns run(n_seqs) -> (seconds, bytes, n_seqs): the oracle doing the
    step for the first n_seqs sequences (their new tokens' writes into a copy
    of the pool, then their decode rows over all heads)."""
    import oracle
    kp0 = workloads.to_numpy_raw(vals["k_pool"])
    vp0 = workloads.to_numpy_raw(vals["v_pool"])
    key = workloads.to_numpy_raw(vals["new_key"])
    value = workloads.to_numpy_raw(vals["new_value"])
    q = workloads.to_numpy_raw(vals["q"])
    assert batch.query_start_loc is None and batch.cow_pairs.shape[0] == 0
    e = elem_bytes(wl.dtype)

    def run(n):
        kp, vp = kp0.copy(), vp0.copy()
        t0 = time.perf_counter()
        oracle.reshape_and_cache(kp, vp, key[:n], value[:n], batch.slot_mapping[:n], wl.dtype)
        oracle.decode(q, kp, vp, batch.block_tables, batch.context_lens, wl.scale, wl.dtype,
                      rows=range(n), threads=host_cores())
        dt = time.perf_counter() - t0
        dec, _, _ = seq_bytes(wl, batch, range(n))
        nbytes = dec + 2 * (2 * n * wl.num_kv_heads * wl.head_dim * e) + n * 8
        return dt, nbytes, n

    return run, host_cores()


def size_sample(run, total, target_s):
    """Pick the number of sequences whose oracle step takes about target_s."""
    n = min(8, total)
    dt, _, _ = run(n)
    while dt < 0.2 * target_s and n < total:
        n = min(total, n * 4)
        dt, _, _ = run(n)
    n = int(min(total, max(1, n * target_s / max(dt, 1e-6))))
    return n


def oracle_config_leg(db, gpu_out, target_s=1.5):
    """The oracle on a sample of one workload's query rows, on the same
    inputs as the GPU call (copy-on-write copies and this step's K/V applied
    to a host copy of the pool first): seconds with all threads (and with one
    thread for the first three workloads), the equivalent GB/s, and the largest
    differences between the sampled rows and the GPU's output."""
    import oracle
    wl, batch, vals = db.wl, db.batch, db.vals
    if db.kv_fp8:
        kp, vp = db.k_codes.numpy(), db.v_codes.numpy()   # host arrays, not on the device
        if batch.cow_pairs.shape[0]:
            oracle.copy_blocks(kp, vp, batch.cow_pairs, "fp8")
        oracle.reshape_and_cache_fp8(kp, vp, workloads.to_numpy_raw(vals["new_key"]),
                                     workloads.to_numpy_raw(vals["new_value"]), wl.dtype,
                                     batch.slot_mapping, db.ks, db.vs)
    else:
        kp = workloads.to_numpy_raw(vals["k_pool"])  # in place: the device pool is a copy
        vp = workloads.to_numpy_raw(vals["v_pool"])
        if batch.cow_pairs.shape[0]:
            oracle.copy_blocks(kp, vp, batch.cow_pairs, wl.dtype)
        oracle.reshape_and_cache(kp, vp, workloads.to_numpy_raw(vals["new_key"]),
                                 workloads.to_numpy_raw(vals["new_value"]), batch.slot_mapping,
                                 wl.dtype)
    q = workloads.to_numpy_raw(vals["q"])
    qsl = batch.query_start_loc
    cores = host_cores()  # every run names its thread count: OpenMP keeps the last one set

    def decode(rows, threads):
        t0 = time.perf_counter()
        if db.kv_fp8:
            ref = oracle.decode_fp8(q, wl.dtype, kp, vp, db.ks, db.vs, batch.block_tables,
                                    batch.context_lens, wl.scale, query_start_loc=qsl, rows=rows,
                                    threads=threads)
        else:
            ref = oracle.decode(q, kp, vp, batch.block_tables, batch.context_lens, wl.scale,
                                wl.dtype, query_start_loc=qsl, rows=rows, threads=threads)
        return time.perf_counter() - t0, ref

    # visible keys of every query row, to size the sample by work
    lens = batch.context_lens.astype(np.int64)
    if qsl is None:
        keys = lens
        row_seq = np.arange(batch.num_seqs)
    else:
        keys, row_seq = [], []
        for i in range(batch.num_seqs):
            Q = int(qsl[i + 1] - qsl[i])
            keys.extend(int(lens[i]) - Q + t + 1 for t in range(Q))
            row_seq.extend([i] * Q)
        keys, row_seq = np.asarray(keys), np.asarray(row_seq)
    order = np.random.default_rng(7).permutation(keys.shape[0])
    probe = order[: max(1, min(8, keys.shape[0]))]
    dt, _ = decode(probe.tolist(), cores)
    per_key = dt / max(1, int(keys[probe].sum()))
    csum = np.cumsum(keys[order])
    n = int(np.searchsorted(csum, target_s / max(per_key, 1e-12))) + 1
    rows = np.sort(order[: max(1, min(n, keys.shape[0]))])
    dt, ref = decode(rows.tolist(), cores)
    e = elem_bytes(wl.dtype)
    ekv = 1 if db.kv_fp8 else e
    kv_bytes = int(keys[rows].sum()) * 2 * wl.num_kv_heads * wl.head_dim * ekv
    nbytes = kv_bytes + 2 * rows.shape[0] * wl.num_heads * wl.head_dim * e
    g = gpu_out.float().cpu().numpy().astype(np.float64)[rows]
    r = ref[rows]
    err = np.abs(g - r)
    big = np.abs(r) > 1e-3
    leg = {"rows": int(rows.shape[0]), "of_rows": int(keys.shape[0]),
           "sample": "query rows drawn uniformly at random (seed 7), all heads; GB/s counts the "
                     "KV bytes each sampled row reads (no sharing between rows)",
           "threads_all": {"cores": cores, "s": dt, "GBps": nbytes / dt / 1e9},
           "max_abs_err_vs_gpu": float(err.max()),
           "max_rel_err_vs_gpu_ref_gt_1e-3": float((err[big] / np.abs(r[big])).max()) if big.any() else 0.0}
    if db.cfg in ("1", "2", "3"):
        rows1 = rows[: max(1, rows.shape[0] // 8)]
        dt1, _ = decode(rows1.tolist(), 1)
        kb1 = int(keys[rows1].sum()) * 2 * wl.num_kv_heads * wl.head_dim * ekv + \
            2 * rows1.shape[0] * wl.num_heads * wl.head_dim * e
        leg["threads_1"] = {"rows": int(rows1.shape[0]), "s": dt1, "GBps": kb1 / dt1 / 1e9}
    return leg


def run_reference(args):
    """--impl reference: the CPU oracle, as it stands, on the host cores."""
    wl = workloads.make(args.config)
    batch = build_batch(wl)
    vals = workloads.values(wl)
    run, cores = oracle_runner(wl, vals, batch)
    n = size_sample(run, batch.num_seqs, target_s=4.0)
    for _ in range(args.warmup):
        run(n)
    times, nbytes = [], 0
    for _ in range(args.steps):
        dt, nbytes, _ = run(n)
        times.append(dt)
    total = sum(times)
    value = nbytes * args.steps / total / 1e9
    sample = (f"first {n} of {batch.num_seqs} sequences per step (their reshape_and_cache writes "
              f"and decode rows, all {wl.num_heads} heads)")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": wl.name, "sample": sample},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# --------------------------------------------------------------------------
# GPU leg
# --------------------------------------------------------------------------
def e2e_pipelined(db, k, warmup, barrier):
    """The step through the public API from page-locked host buffers: every
    step copies its inputs in (q, new K/V, slots, context lengths and the
    block-table entries the step appended) and its output back; copies of
    neighbouring steps overlap the kernels (PagedKVCache
    .capture_pipelined_steps_from_host)."""
    from paged_kv_cache_388_b200.session import PagedKVCache
    wl, batch, vals = db.wl, db.batch, db.vals
    idx, ids = PagedKVCache.appended_table_entries(batch.block_tables, batch.context_lens,
                                                   wl.block_size)
    host = {"q": vals["q"].pin_memory(), "key": vals["new_key"].pin_memory(),
            "value": vals["new_value"].pin_memory(),
            "slot_mapping": torch.from_numpy(batch.slot_mapping).pin_memory(),
            "context_lens": torch.from_numpy(batch.context_lens).pin_memory(),
            "bt_index": idx.pin_memory(), "bt_ids": ids.pin_memory()}
    outs = [torch.empty_like(host["q"]).pin_memory() for _ in range(2)]
    steps = [dict(host, out=outs[i % 2]) for i in range(k)]
    replay = db.cache.capture_pipelined_steps_from_host(steps, db.bt, wl.scale,
                                                        max_context_len=db.mcl, warmup=1)
    for _ in range(max(1, warmup // 2)):
        replay()
    stream = torch.cuda.current_stream(db.dev)
    # the median of five timed replays of the K steps (the host side of the
    # copies sees other work on the machine; one replay is exposed to a stall)
    times = []
    for _ in range(5):
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        replay()
        e1.record(stream)
        barrier()
        times.append(e0.elapsed_time(e1))
    h2d = PagedKVCache.host_bytes(*host.values())
    d2h = PagedKVCache.host_bytes(outs[0])
    ms = float(np.median(times))
    assert torch.equal(outs[(k - 1) % 2], db.out.cpu()), "end-to-end output differs from the device step"
    return ms, h2d, d2h, (min(times), max(times))


def run_ours(args, rank, world, local_rank):
    import torch.distributed as dist

    from paged_kv_cache_388_b200 import _lib

    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    timer = Timer(dev)
    stream = timer.stream
    K = args.steps

    # weak scaling: every rank runs its own batch of the workload's shape
    db = DeviceBatch(args.config, dev, replica=rank, kv_fp8=args.kv_fp8,
                     plain_decode=args.plain_decode)
    wl, batch, nbytes = db.wl, db.batch, db.bytes
    launches_per_step = db.launches_per_step()

    for _ in range(args.warmup):  # eager warm-up: one-time library set-up
        db.step()
    torch.cuda.synchronize(dev)
    assert _lib.pa_get_device_error() == 0

    # The K timed steps are captured into one CUDA graph (no host launch
    # overhead between kernels).
    g_steps = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_steps):
        for _ in range(K):
            db.step()
    g_warm = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_warm):
        db.step()
    for _ in range(args.warmup):
        g_warm.replay()
    torch.cuda.synchronize(dev)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    # The clock record spans the timed steps and the per-call timings that
    # the roofline figures come from (the K steps alone last a few ms, less
    # than the sampling period).
    with ClockSampler(local_rank) as clocks:
        barrier()
        t_start.record(stream)
        g_steps.replay()
        t_end.record(stream)
        barrier()
        ms_local = t_start.elapsed_time(t_end)
        job_bytes, ms = aggregate(nbytes["step"] * K, ms_local, dev)
        assert _lib.pa_get_device_error() == 0
        del g_steps, g_warm

        # per-call device time of the step's calls: K back-to-back calls in one
        # graph (inputs larger than L2) and 50 single calls after an L2 flush
        dec_avg = timer.back_to_back(db.attend, K)
        res_avg = timer.back_to_back(db.write, K)
        dec_flushed = timer.flushed(db.attend)
        torch.cuda.synchronize(dev)
    clk = clocks.summary()
    clk["window"] = "timed steps and the per-call timings of the step's calls"

    # ---- end to end through the public API, host (pinned) buffers ----------
    e2e = None
    if batch.query_start_loc is None and db.cow.shape[0] == 0 and not db.shared:
        e2e_ms, h2d, d2h, (e2e_lo, e2e_hi) = e2e_pipelined(db, K, args.warmup, barrier)
        e2e_bytes, e2e_ms = aggregate(nbytes["step"] * K, e2e_ms, dev)
        e2e = {"value": e2e_bytes / (e2e_ms * 1e-3) / 1e9, "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / K,
               "ms_per_step_min_max": [e2e_lo / K, e2e_hi / K],
               "timing": "median of 5 timed replays of the K-step graph (max over ranks)",
               "path": "PagedKVCache.capture_pipelined_steps_from_host (CUDA graph of K steps; "
                       "H2D and D2H copies on their own streams overlap the neighbouring steps' "
                       "kernels; block tables resident, appended entries sent per step)"}

    # ---- every other workload, call by call (one GPU) ----------------------
    configs = {}
    if world == 1 and not args.headline_only:
        configs[args.config + ("fp8" if args.kv_fp8 else "")] = measure_config(db, timer, K)
    head_out = db.out.clone()

    # ---- CPU oracle baseline on a bounded sample (rank 0, N = 1) -----------
    cpu = None
    if (rank == 0 and world == 1 and not args.no_cpu_baseline and batch.query_start_loc is None
            and not args.kv_fp8 and batch.cow_pairs.shape[0] == 0):
        run, cores = oracle_runner(wl, db.vals, batch)
        n = size_sample(run, batch.num_seqs, target_s=8.0)
        dt, ob, _ = run(n)
        cpu = {"value": ob / dt / 1e9, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"first {n} of {batch.num_seqs} sequences (reshape_and_cache of their "
                         f"new tokens + decode rows over all {wl.num_heads} heads), "
                         f"one run of {dt:.1f} s"}
        cpu["per_config"] = {}
        if configs:
            cpu["per_config"][args.config] = oracle_config_leg(db, head_out)

    if world == 1 and not args.headline_only:
        del db
        gc.collect()
        torch.cuda.empty_cache()
        for cfg in (args.extra_configs.split(",") if args.extra_configs else EXTRA_CONFIGS):
            if not cfg or cfg == args.config:
                continue
            fp8 = cfg.endswith("fp8")
            xdb = DeviceBatch(cfg[:-3] if fp8 else cfg, dev, kv_fp8=fp8)
            configs[cfg] = measure_config(xdb, timer, K)
            assert _lib.pa_get_device_error() == 0
            if cpu is not None:
                cpu["per_config"][cfg] = oracle_config_leg(xdb, xdb.out)
            del xdb
            gc.collect()
            torch.cuda.empty_cache()
    else:
        del db

    peak, peak_kind = hbm_peak()
    achieved = nbytes["decode"] / (dec_avg * 1e-3) / 1e9
    value = job_bytes / (ms * 1e-3) / 1e9
    call_name = (("pa_decode_shared_prefix" if args.config.startswith("4") and not args.plain_decode
                  else "pa_decode") + ("_fp8" if args.kv_fp8 else ""))
    res = {
        "metric": METRIC,
        "value": value,
        "unit": UNIT,
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": ("fp8_e4m3 KV cache, " + wl.dtype + " q/out") if args.kv_fp8 else wl.dtype,
        "data": "synthetic",
        "config": {
            "workload": wl.name + ("_kv_fp8_e4m3" if args.kv_fp8 else ""),
            "global_batch": batch.num_seqs * world,
            "heads": f"{wl.num_heads}q/{wl.num_kv_heads}kv",
            "head_dim": wl.head_dim,
            "block_size": wl.block_size,
            "kv_tokens": nbytes["kv_tokens"],
            "step_bytes": nbytes["step"],
            "l2": f"inputs larger than L2 ({nbytes['decode'] / 1e9:.2f} GB of KV per step vs "
                  f"{L2_BYTES / 2**20:.0f} MiB L2); no flush in the timed steps; per-call "
                  f"medians flush L2 before every call",
            "parallelism": f"dp{world} (independent batches)",
        },
        "decode_tokens_per_s": batch.num_seqs * world * K / (ms * 1e-3),
        "pct_of_nominal_8TBps": 100.0 * value / NOMINAL_HBM_GBS,
        "roofline": {
            "kernel": f"{call_name} (paged_decode_mma_kernel + balanced_merge_kernel)",
            "bound": "hbm",
            "achieved": achieved,
            "peak": peak,
            "peak_kind": f"{peak_kind} copy bandwidth",
            "unit": "GB/s",
            "frac": achieved / peak,
            "frac_of_nominal_8TBps": achieved / NOMINAL_HBM_GBS,
            "traffic": None if args.kv_fp8 else profiled_traffic(args.config),
            "traffic_source": "profiles/paged_decode_mma_kernel_cfg3.md (ncu dram__bytes_read+write "
                              "of the decode kernel; null when the kernel sources changed since)",
            "algorithmic_bytes": nbytes["decode"],
            "avg_ms": dec_avg,
            "flushed_calls": dec_flushed,
        },
        "kernels_ms": {call_name: dec_avg, "pa_reshape_and_cache": res_avg},
        "cpu_baseline": cpu,
        "e2e": e2e,
        **({"configs": configs} if configs else {}),
        "gpu_launches": launches_per_step * K,
        "clocks": clk,
    }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return res


def run_swap(args):
    """Swap-out / swap-in of KV blocks between the device pool and a pinned
    host pool (pa_swap_blocks), against the host link's DMA copy rate."""
    from paged_kv_cache_388_b200.session import PagedKVCache

    dev = torch.device("cuda", 0)
    wl = workloads.make(args.config)
    batch = build_batch(wl)
    vals = workloads.values(wl)
    cache = PagedKVCache(wl.num_blocks, wl.num_kv_heads, wl.head_dim, wl.block_size,
                         k_cache=vals["k_pool"].to(dev), v_cache=vals["v_pool"].to(dev))
    # preempt the first half of the sequences: every block they hold goes out
    half = batch.num_seqs // 2
    blocks = []
    for i in range(half):
        n = -(-int(batch.context_lens[i]) // wl.block_size)
        blocks.extend(int(b) for b in batch.block_tables[i, :n])
    blocks = np.unique(np.asarray(blocks, dtype=np.int64))
    nb = blocks.shape[0]
    host_k, host_v = cache.host_pool(nb)
    out_map = torch.from_numpy(np.stack([blocks, np.arange(nb)], 1)).to(dev)
    in_map = out_map.flip(1).contiguous()
    block_bytes = 2 * wl.num_kv_heads * wl.block_size * wl.head_dim * elem_bytes(wl.dtype)
    nbytes = nb * block_bytes
    stream = torch.cuda.current_stream(dev)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / args.steps

    ms_out = timed(lambda: cache.swap_out(host_k, host_v, out_map))
    ms_in = timed(lambda: cache.swap_in(host_k, host_v, in_map))
    # the host link's DMA rate on the same bytes (one contiguous copy each way)
    hbuf = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    dbuf = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    ms_h2d = timed(lambda: dbuf.copy_(hbuf, non_blocking=True))
    ms_d2h = timed(lambda: hbuf.copy_(dbuf, non_blocking=True))
    gb = lambda ms: nbytes / (ms * 1e-3) / 1e9  # noqa: E731
    return {
        "metric": "KV block swap between device pool and pinned host pool (pa_swap_blocks)",
        "value": gb(ms_out + ms_in) * 2, "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "dtype": wl.dtype, "data": "synthetic",
        "config": {"workload": wl.name, "blocks": int(nb), "bytes_per_direction": int(nbytes),
                   "block_bytes": block_bytes, "pairs_scattered": True},
        "swap_out": {"ms": ms_out, "GBps": gb(ms_out)},
        "swap_in": {"ms": ms_in, "GBps": gb(ms_in)},
        "roofline": {"bound": "host link", "peak_d2h_GBps": gb(ms_d2h), "peak_h2d_GBps": gb(ms_h2d),
                     "peak_kind": "measured contiguous DMA copy of the same bytes (cudaMemcpyAsync)",
                     "frac_out": ms_d2h / ms_out, "frac_in": ms_h2d / ms_in},
        "gpu_launches": 2 * args.steps,
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="3")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the per-workload call timings (the `configs` block)")
    ap.add_argument("--extra-configs", default="",
                    help="comma-separated workloads for the `configs` block (default: all)")
    ap.add_argument("--plain-decode", action="store_true",
                    help="attend shared-prefix batches with pa_decode instead of "
                         "pa_decode_shared_prefix")
    ap.add_argument("--memory-report", action="store_true",
                    help="host only: KV slots held by paged blocks vs max-length reservation")
    ap.add_argument("--kv-fp8", action="store_true",
                    help="FP8 (E4M3) KV cache: pa_reshape_and_cache_fp8 + pa_decode_fp8")
    ap.add_argument("--swap", action="store_true",
                    help="time pa_swap_blocks (device <-> pinned host) instead of the decode step")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.swap:
        print(json.dumps(run_swap(args)), flush=True)
        return
    if args.memory_report:
        from paged_kv_cache_388_b200.memory import pool_usage, waste_report
        for cfg, max_len in (("1", 100), ("2", 2048), ("3", 4096), ("4", 1536), ("4cow", 1528),
                             ("5", 131072), ("5bs32", 131072)):
            wl = workloads.make(cfg)
            rep = waste_report(wl.seq_context_lens(), wl.block_size, max_len)
            rep["pool"] = pool_usage(build_batch(wl).allocator)
            print(json.dumps({"config": wl.name, "reservation_len": max_len, **rep}), flush=True)
        return

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    res = run_ours(args, rank, world, local_rank)
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
