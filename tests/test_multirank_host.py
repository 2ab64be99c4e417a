"""Multi-rank host logic on CPU (gloo, world size 2): every rank builds its own
replica batch of the workload (weak scaling, no collective on the data path)
and the benchmark's aggregation sums bytes and takes the slowest rank's time."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import workloads
        from paged_kv_cache_388_b200.batch import build_batch
        wl = workloads.make("3s", replica=rank)
        b = build_batch(wl)
        local = bench.step_bytes(wl, b)["step"]
        ms = 10.0 + rank  # stand-in device times
        total, mx = bench.aggregate(local, ms, "cpu")
        lens = torch.tensor(b.context_lens.astype(np.int64))
        gathered = [torch.zeros_like(lens) for _ in range(world)]
        dist.all_gather(gathered, lens)
        out[rank] = (local, total, mx, [g.tolist() for g in gathered])
    finally:
        dist.destroy_process_group()


def test_two_rank_weak_scaling_aggregation():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    locals_ = [out[r][0] for r in range(world)]
    for r in range(world):
        _, total, mx, lens = out[r]
        assert total == sum(locals_)        # bytes of all ranks
        assert mx == 10.0 + (world - 1)     # slowest rank's time
        assert lens[0] != lens[1]           # each rank runs its own batch
