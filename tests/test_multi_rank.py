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


# ---------------------------------------------------------------------------
# LPT head sharding of one model over ranks (strong scaling) and the gather
# of the ranks' varlen packed outputs into head order.
# ---------------------------------------------------------------------------

def _model_budgets():
    sys.path.insert(0, ROOT)
    from attention_matching_b200 import workloads as W
    return W.lognormal_budgets(4999, 288, 47186)


def test_lpt_partition_covers_every_head_once_and_balances():
    sys.path.insert(0, ROOT)
    from attention_matching_b200.sharding import head_cost, lpt_partition
    budgets = _model_budgets()
    costs = [head_cost(t, 8) for t in budgets]
    for world in (1, 2, 4, 8):
        parts = lpt_partition(costs, world)
        assert sorted(h for p in parts for h in p) == list(range(288))
        assert all(p == sorted(p) for p in parts)
        loads = [sum(costs[h] for h in p) for p in parts]
        # LPT: no rank exceeds the average by more than the largest single cost
        assert max(loads) <= sum(costs) / world + max(costs)
        assert parts == lpt_partition(costs, world)           # deterministic
    # by hand: costs 5, 4, 3, 3, 3 over two ranks; 5 -> r0, 4 -> r1, head 2 -> r1
    # (load 4 < 5), head 3 -> r0 (5 < 7), head 4 -> r1 (7 < 8)
    assert lpt_partition([5, 4, 3, 3, 3], 2) == [[0, 3], [1, 2, 4]]
    assert head_cost(164, 8) == 164 * 21 and head_cost(8, 8) == 8


def _gather_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    from attention_matching_b200.sharding import gather_packed, head_cost, lpt_partition
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        budgets = [3, 1, 4, 1, 5, 9, 2, 6]
        d = 4
        parts = lpt_partition([head_cost(t, 2) for t in budgets], world)
        mine = parts[rank]
        rows = sum(budgets[h] for h in mine)
        # head h's row r carries (h, r) so the assembled order can be read back
        Ck = torch.tensor([[h, r, 0, 0] for h in mine for r in range(budgets[h])], dtype=torch.float32)
        local = {"C_k": Ck.to(torch.bfloat16), "beta": Ck[:, 0] * 10 + Ck[:, 1],
                 "C_v": Ck + 0.5, "indices": Ck[:, 1].to(torch.int32)}
        assert local["C_k"].shape == (rows, d)
        g = gather_packed(local, mine, budgets, dist)
        out[rank] = {k: v.float().tolist() if k != "cu_t" else v.tolist() for k, v in g.items()}
    finally:
        dist.destroy_process_group()


def test_gather_packed_outputs_into_head_order_two_gloo_ranks():
    world = 2
    port = _free_port()
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_gather_main, args=(world, port, out), nprocs=world, join=True)
    budgets = [3, 1, 4, 1, 5, 9, 2, 6]
    want_rows = [(h, r) for h in range(len(budgets)) for r in range(budgets[h])]
    for rank in range(world):
        g = out[rank]
        assert g["cu_t"] == [0, 3, 4, 8, 9, 14, 23, 25, 31]
        assert [(int(a), int(b)) for a, b, _, _ in g["C_k"]] == want_rows
        assert g["beta"] == [10.0 * h + r for h, r in want_rows]
        assert g["indices"] == [float(r) for _, r in want_rows]
        assert g["C_v"][5] == [want_rows[5][0] + 0.5, want_rows[5][1] + 0.5, 0.5, 0.5]
