"""Multi-process host paths on CPU (gloo, world size 2): the sharded tie-group amax
all-reduce, and the benchmark's max-over-ranks timing and weak-scaling aggregate."""
import os
import socket

import numpy as np
import pytest
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
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import workloads
        from fp4_fake_quant_b200.distributed import fold_tracked, reduce_group_amax
        # each rank holds a shard (half the rows) of every tensor of two tie groups
        wl = workloads.nvfp4_tied(rows_scale=1 / 64, with_grads=False)
        shards = [t[rank * (t.shape[0] // world):(rank + 1) * (t.shape[0] // world)]
                  for t in wl["tensors"]]
        local = torch.from_numpy(oracle.tied_amax(shards, wl["groups"], 2))
        reduce_group_amax(local)
        full = oracle.tied_amax([t[: (t.shape[0] // world) * world] for t in wl["tensors"]],
                                wl["groups"], 2)
        ok_amax = bool(np.array_equal(local.numpy().view(np.uint32), full.view(np.uint32)))
        # a tracked amax above the step's amax in group 0 and below it in group 1: both
        # ranks end with tracked = max(tracked, global amax) and quantize with it
        tracked = torch.tensor([float(full[0]) * 2, float(full[1]) / 2], dtype=torch.float32)
        want = np.maximum(tracked.numpy(), full)
        fold_tracked(local, tracked)
        ok_amax &= bool(np.array_equal(tracked.numpy(), want) and np.array_equal(local.numpy(), want))
        # the benchmark's aggregation: max over ranks of each device time, and the
        # whole-job value = world x bytes per step / slowest step
        import bench
        total, kern = bench.max_over_ranks([10.0 + rank, 1.0 + 2 * rank], "cpu")
        ok_time = (total, kern) == (10.0 + world - 1, 1.0 + 2 * (world - 1))
        ok_value = bench.weak_scaling_value(1e9, world, total) == world * 1e9 / (total * 1e-3) / 1e9
        # ranks draw different seeded batches (seed shifted by 1000 per rank)
        a = workloads.mxfp4_w4a4(rows_scale=1 / 1024, seed=1 + 1000 * rank)["tensors"][0]
        g = [torch.zeros_like(a) for _ in range(world)]
        dist.all_gather(g, a)
        ok_seed = not torch.equal(g[0], g[1])
        out[rank] = (ok_amax, ok_time, ok_seed, ok_value)
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_sharded_amax_and_timing():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    port = _free_port()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        assert out[r] == (True, True, True, True), (r, out[r])
