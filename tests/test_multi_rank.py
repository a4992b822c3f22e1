"""The multi-GPU bench path on CPU: two gloo ranks run the same cross-rank
steps bench.py takes (max-over-ranks step time, whole-job throughput, a
distinct seeded workload per rank); no GPU is involved."""
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_ms = 10.0 + 5.0 * rank                       # rank 1 is the slow one
        ms = bench.max_over_ranks(my_ms, dist, "cpu")
        wl = bench.build_workload("single_head_fp32", rank)
        key0 = float(wl.heads[0].K[0, 0])
        keys = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(keys, torch.tensor([key0], dtype=torch.float64))
        out[rank] = (ms, bench.job_throughput(len(wl.heads), world, ms), [float(k) for k in keys])
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_job_time_and_throughput():
    world = 2
    port = _free_port()
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        ms, value, keys = out[r]
        assert ms == 15.0                               # the max over ranks, on every rank
        assert abs(value - 1 * world / 15e-3) < 1e-9    # weak scaling: heads of all ranks / job time
        assert keys[0] != keys[1]                       # each rank compacts its own seeded heads


def test_single_process_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(12.5, None, "cpu") == 12.5
    assert bench.job_throughput(8, 1, 20.0) == 400.0
