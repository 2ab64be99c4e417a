#!/usr/bin/env python
"""Benchmark: one decode step of paged attention on the Llama-3-8B-shaped GQA batch.

A step is the whole hot path over one batch: copy-on-write block copies (none
in this batch), reshape_and_cache of the step's 256 new tokens, then paged
decode attention of the 256 query tokens over their block-table KV cache
(32 query heads / 8 KV heads, head_dim 128, block size 16, bf16, context
lengths lognormal with median 800 capped at 4096, shuffled pool).

Printed (rank 0, one JSON line): achieved HBM GB/s of the step (algorithmic
bytes / device time), decode tokens/s, the dominant kernel's roofline, an
end-to-end figure through the public API with host buffers, and the CPU oracle
timed on a bounded sample as a baseline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 is launched with torchrun: every rank runs its own batch (weak scaling,
no collective on the data path); times are the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
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
from paged_kv_cache_388_b200.batch import build_batch, shared_prefix_groups  # noqa: E402

METRIC = "paged decode attention: achieved HBM GB/s (% of peak) and decode tokens/s"
UNIT = "GB/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 2 ** 20


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


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


def tensor_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


def chunk_flops(batch):
    """Multiply-add FLOPs of the chunked-query rows (QK^T and PV over the keys
    each row may see): sum over rows of visible keys * H * D * 4."""
    qsl = batch.query_start_loc
    if qsl is None:
        return 0
    total = 0
    for i, L in enumerate(batch.context_lens.tolist()):
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


# --------------------------------------------------------------------------
# CPU oracle legs (cpu_baseline and --impl reference)
# --------------------------------------------------------------------------
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
                      rows=range(n))
        dt = time.perf_counter() - t0
        dec, _, _ = seq_bytes(wl, batch, range(n))
        nbytes = dec + 2 * (2 * n * wl.num_kv_heads * wl.head_dim * e) + n * 8
        return dt, nbytes, n

    return run, oracle.max_threads()


def size_sample(run, total, target_s):
    """Pick the number of sequences whose oracle step takes about target_s."""
    n = min(8, total)
    dt, _, _ = run(n)
    while dt < 0.2 * target_s and n < total:
        n = min(total, n * 4)
        dt, _, _ = run(n)
    n = int(min(total, max(1, n * target_s / max(dt, 1e-6))))
    return n


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
def run_ours(args, rank, world, local_rank):
    import torch.distributed as dist

    from paged_kv_cache_388_b200 import _lib
    from paged_kv_cache_388_b200.session import PagedKVCache

    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)

    # weak scaling: every rank runs its own batch of the workload's shape
    wl = workloads.make(args.config, replica=rank)
    batch = build_batch(wl)
    vals = workloads.values(wl)
    nbytes = step_bytes(wl, batch, 1 if args.kv_fp8 else None)

    if args.kv_fp8:
        # FP8 (E4M3) cache: one scale per tensor, the pool's history quantised
        # on the host, this step's K/V quantised by pa_reshape_and_cache_fp8
        def fp8_scale(*ts):
            return float(np.float32(max(float(t.float().abs().max()) for t in ts) / 448.0 * 1.25))

        def quant(t, sc):
            return (t.float() / torch.tensor(sc, dtype=torch.float32)).to(
                torch.float8_e4m3fn).view(torch.uint8)

        ks = fp8_scale(vals["k_pool"], vals["new_key"])
        vs = fp8_scale(vals["v_pool"], vals["new_value"])
        cache = PagedKVCache(wl.num_blocks, wl.num_kv_heads, wl.head_dim, wl.block_size,
                             dtype=torch.uint8, k_cache=quant(vals["k_pool"], ks).to(dev),
                             v_cache=quant(vals["v_pool"], vs).to(dev), kv_scales=(ks, vs))
    else:
        cache = PagedKVCache(wl.num_blocks, wl.num_kv_heads, wl.head_dim, wl.block_size,
                             k_cache=vals["k_pool"].to(dev), v_cache=vals["v_pool"].to(dev))
    q = vals["q"].to(dev)
    key = vals["new_key"].to(dev)
    value = vals["new_value"].to(dev)
    slot = torch.from_numpy(batch.slot_mapping).to(dev)
    bt = torch.from_numpy(batch.block_tables).to(dev)
    cl = torch.from_numpy(batch.context_lens).to(dev)
    qsl = None if batch.query_start_loc is None else torch.from_numpy(batch.query_start_loc).to(dev)
    cow = torch.from_numpy(np.ascontiguousarray(batch.cow_pairs)).to(dev)
    out = torch.empty_like(q)
    mcl = batch.max_context_len
    ws_bytes = _lib.pa_decode_workspace_size(batch.num_seqs, wl.num_heads, wl.num_kv_heads,
                                             wl.head_dim, wl.block_size, mcl, 0)
    cache.workspace(batch.num_seqs, wl.num_heads, mcl)
    stream = torch.cuda.current_stream(dev)

    # Batches whose sequences share prompt blocks (parallel sampling) attend
    # through the shared-prefix entry point unless --plain-decode is given.
    shared = wl.kind == "shared_prefix" and not args.plain_decode and not args.kv_fp8
    if shared:
        gs_np, gb_np = shared_prefix_groups(batch.block_tables, batch.context_lens, wl.block_size)
        gs = torch.from_numpy(gs_np).to(dev)
        gb = torch.from_numpy(gb_np).to(dev)
        max_group = int(np.diff(gs_np).max())

    def attend_plain():
        cache.attend(q, bt, cl, wl.scale, out=out, query_start_loc=qsl,
                     max_query_len=batch.max_query_len, max_context_len=mcl)

    def attend():
        if shared:
            cache.attend_shared_prefix(q, bt, cl, gs, gb, wl.scale, max_group_size=max_group,
                                       out=out, max_context_len=mcl)
        else:
            attend_plain()

    K = args.steps

    def step(evs=None):
        if cow.shape[0]:
            cache.copy_blocks(cow)
        if evs:
            evs[0].record(stream)
        cache.write(key, value, slot)
        if evs:
            evs[1].record(stream)
        attend()
        if evs:
            evs[2].record(stream)

    for _ in range(args.warmup):  # eager warm-up: one-time library set-up
        step()
    torch.cuda.synchronize(dev)
    assert _lib.pa_get_device_error() == 0

    # The K timed steps are captured into one CUDA graph (no host launch
    # overhead between kernels).
    g_steps = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_steps):
        for _ in range(K):
            step()
    g_warm = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_warm):
        step()
    for _ in range(args.warmup):
        g_warm.replay()
    torch.cuda.synchronize(dev)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clocks:
        barrier()
        t_start.record(stream)
        g_steps.replay()
        t_end.record(stream)
        barrier()
    ms_local = t_start.elapsed_time(t_end)
    job_bytes, ms = aggregate(nbytes["step"] * K, ms_local, dev)
    assert _lib.pa_get_device_error() == 0
    clk = clocks.summary()
    del g_steps, g_warm

    # Per-call device time of the step's two calls, each timed as K back-to-back
    # calls in its own CUDA graph (CUDA events on the launching stream).
    def time_graph(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(K):
                fn()
        g.replay()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / K

    dec_avg = time_graph(attend)
    res_avg = time_graph(lambda: cache.write(key, value, slot))

    # Mixed batches: the decode rows and the chunked-query rows, each timed alone
    parts = {}
    if shared:  # the same batch through plain decode (every shared block read per sequence)
        plain_ms = time_graph(attend_plain)
        logical = sum(int(batch.context_lens[i]) for i in range(batch.num_seqs)) * 2 * \
            wl.num_kv_heads * wl.head_dim * elem_bytes(wl.dtype)
        parts["plain_decode"] = {"ms": plain_ms,
                                 "GBps_unique": nbytes["decode"] / (plain_ms * 1e-3) / 1e9}
        parts["shared_prefix"] = {"ms": dec_avg,
                                  "GBps_unique": nbytes["decode"] / (dec_avg * 1e-3) / 1e9,
                                  "groups": int(gb_np.shape[0]),
                                  "shared_blocks": int(gb_np.max()),
                                  "logical_kv_bytes": logical}
    if batch.query_start_loc is not None:
        qsl_np = batch.query_start_loc
        dec_ids = [i for i in range(batch.num_seqs) if qsl_np[i + 1] - qsl_np[i] == 1]
        chk_ids = [i for i in range(batch.num_seqs) if qsl_np[i + 1] - qsl_np[i] > 1]
        for name, ids in (("decode_rows", dec_ids), ("chunk_rows", chk_ids)):
            if not ids:
                continue
            sbt, scl, sqsl, srows = sub_batch(batch, ids)
            sq = q[torch.from_numpy(srows).to(dev)].contiguous()
            sout = torch.empty_like(sq)
            t_bt = torch.from_numpy(np.ascontiguousarray(sbt)).to(dev)
            t_cl = torch.from_numpy(np.ascontiguousarray(scl)).to(dev)
            t_qsl = None if sqsl is None else torch.from_numpy(sqsl).to(dev)
            mql = int(max(np.diff(sqsl))) if sqsl is not None else 1
            if t_qsl is not None and mql == 1:
                t_qsl = None
            parts[name] = {"ms": time_graph(lambda: cache.attend(
                sq, t_bt, t_cl, wl.scale, out=sout, query_start_loc=t_qsl, max_query_len=mql,
                max_context_len=int(scl.max())))}
        if "decode_rows" in parts:
            dbytes, _, _ = seq_bytes(wl, batch, dec_ids)
            parts["decode_rows"]["GBps"] = dbytes / (parts["decode_rows"]["ms"] * 1e-3) / 1e9
        if "chunk_rows" in parts:
            fl = chunk_flops(batch) * wl.num_heads * wl.head_dim * 4
            parts["chunk_rows"]["flops"] = fl
            parts["chunk_rows"]["TFLOPs"] = fl / (parts["chunk_rows"]["ms"] * 1e-3) / 1e12

    # ---- end to end through the public API, host (pinned) buffers ----------
    hq = vals["q"].pin_memory()
    hkey = vals["new_key"].pin_memory()
    hval = vals["new_value"].pin_memory()
    hslot = torch.from_numpy(batch.slot_mapping).pin_memory()
    hbt = torch.from_numpy(batch.block_tables).pin_memory()
    hcl = torch.from_numpy(batch.context_lens).pin_memory()
    hout = torch.empty_like(hq).pin_memory()
    h2d = PagedKVCache.host_bytes(hq, hkey, hval, hslot, hbt, hcl)
    d2h = PagedKVCache.host_bytes(hout)
    e2e_ok = batch.query_start_loc is None and cow.shape[0] == 0 and not shared
    e2e = None
    if e2e_ok:
        # the public API's captured host step: copy in, write K/V, attend, copy out
        replay = cache.capture_step_from_host(hq, hkey, hval, hslot, hbt, hcl, hout, wl.scale,
                                              max_context_len=mcl, warmup=args.warmup)
        for _ in range(args.warmup):
            replay()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(K):
            replay()
        e1.record(stream)
        barrier()
        e2e_bytes, e2e_ms = aggregate(nbytes["step"] * K, e0.elapsed_time(e1), dev)
        e2e = {"value": e2e_bytes / (e2e_ms * 1e-3) / 1e9, "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e2e_ms / K, "path": "PagedKVCache.capture_step_from_host (CUDA graph)"}

    # ---- CPU oracle baseline on a bounded sample (rank 0, N = 1) -----------
    cpu = None
    if (rank == 0 and world == 1 and not args.no_cpu_baseline and batch.query_start_loc is None
            and not args.kv_fp8):
        run, cores = oracle_runner(wl, vals, batch)
        n = size_sample(run, batch.num_seqs, target_s=12.0)
        dt, ob, _ = run(n)
        cpu = {"value": ob / dt / 1e9, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"first {n} of {batch.num_seqs} sequences (reshape_and_cache of their "
                         f"new tokens + decode rows over all {wl.num_heads} heads), "
                         f"one run of {dt:.1f} s"}

    splits = ws_bytes > 0  # the decode call also launches its merge kernel
    launches_per_step = 1 + 1 + (1 if splits else 0) + (1 if cow.shape[0] else 0) + \
        (1 if batch.max_query_len > 1 else 0) + (1 if shared else 0)
    peak, peak_kind = hbm_peak()
    achieved = nbytes["decode"] / (dec_avg * 1e-3) / 1e9
    value = job_bytes / (ms * 1e-3) / 1e9
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
                  f"{L2_BYTES / 2**20:.0f} MiB L2); no flush",
            "parallelism": f"dp{world} (independent batches)",
        },
        "decode_tokens_per_s": batch.num_seqs * world * K / (ms * 1e-3),
        "pct_of_nominal_8TBps": 100.0 * value / NOMINAL_HBM_GBS,
        "roofline": {
            "kernel": ("pa_decode_shared_prefix (shared_prefix_kernel + paged_decode_mma_kernel + "
                       "balanced_merge_kernel)") if shared else
                      "pa_decode (paged_decode_mma_kernel + balanced_merge_kernel)",
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
        },
        "kernels_ms": {("pa_decode_shared_prefix" if shared else "pa_decode"): dec_avg,
                       "pa_reshape_and_cache": res_avg},
        "cpu_baseline": cpu,
        "e2e": e2e,
        **({"parts": parts} if parts else {}),
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
