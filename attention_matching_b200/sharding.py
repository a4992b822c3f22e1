"""Head sharding over GPUs: one process per GPU, each compacting its own
subset of one model's heads; no collective on the data path.

The heads are independent problems ("Fast KV Compaction via Attention
Matching": every (layer, KV head) is compacted on its own, zhichai.net deep
dive §1.6; compaction across GPUs is named as future work, §6.2), so the
only multi-GPU question is balance.  A head's cost is dominated by its OMP
pass chain: ⌈t/(k·R)⌉ passes whose refits and Gram updates grow with the
number of keys already picked, so cost_h = t_h·⌈t_h/(k·R)⌉ (for heads of equal
T and n).  Heads are placed by longest processing time first (LPT): in
descending cost, each to the rank with the smallest load so far.  Outputs
stay on the rank that made them; gather_packed assembles them in head order
for a consumer that needs every head in one place.

This module holds host-side scheduling only: no compaction arithmetic.
"""
from __future__ import annotations

import math
from typing import Dict, List, Sequence


def head_cost(budget: int, picks_per_pass: int) -> int:
    """t_h·⌈t_h / (k·R)⌉: the picks times the passes of one head."""
    return int(budget) * math.ceil(int(budget) / int(picks_per_pass))


def lpt_partition(costs: Sequence[float], world: int) -> List[List[int]]:
    """Heads per rank by LPT: heads in descending cost (ties: lower head
    first) each go to the rank with the least total cost so far (ties: lower
    rank).  Every rank's list is returned in ascending head order."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(costs)), key=lambda h: (-costs[h], h))
    load = [0.0] * world
    parts: List[List[int]] = [[] for _ in range(world)]
    for h in order:
        r = min(range(world), key=lambda q: (load[q], q))
        parts[r].append(h)
        load[r] += costs[h]
    return [sorted(p) for p in parts]


def gather_packed(local: Dict, my_heads: Sequence[int], budgets: Sequence[int], dist) -> Dict:
    """Assemble every rank's packed outputs (C_k, beta, C_v, indices at its
    own cu_t) into one packed set in global head order on every rank.  `local`
    holds this rank's tensors, `my_heads` its heads in the order they were
    packed, `budgets` the budgets of all heads.  Uses all_gather_object (a
    host-side collective for a consumer, not part of the compaction)."""
    import numpy as np
    import torch
    bf16 = local["C_k"].dtype == torch.bfloat16
    # bf16 keys travel as fp32 (exact) and are rounded back, losslessly, after
    mine = {k: (local[k].detach().cpu().float() if k == "C_k" and bf16 else local[k].detach().cpu()).numpy()
            for k in ("C_k", "beta", "C_v", "indices")}
    pieces = [None] * dist.get_world_size()
    dist.all_gather_object(pieces, (list(my_heads), mine))
    cu = np.concatenate([[0], np.cumsum(budgets)]).astype(np.int64)
    total = int(cu[-1])
    d = mine["C_k"].shape[1]
    out = {"C_k": np.zeros((total, d), np.float32), "beta": np.zeros(total, np.float32),
           "C_v": np.zeros((total, d), np.float32), "indices": np.zeros(total, np.int32)}
    seen = np.zeros(len(budgets), bool)
    for heads, arrs in pieces:
        at = 0
        for h in heads:
            t = int(budgets[h])
            for k in out:
                out[k][cu[h]:cu[h + 1]] = arrs[k][at:at + t]
            at += t
            seen[h] = True
    if not seen.all():
        raise ValueError("some heads were compacted on no rank")
    res = {k: torch.from_numpy(v) for k, v in out.items()}
    if bf16:
        res["C_k"] = res["C_k"].to(torch.bfloat16)
    res["cu_t"] = torch.from_numpy(cu)
    return res
