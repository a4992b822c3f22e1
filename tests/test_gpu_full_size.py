"""GPU parity at the full sizes of the pages' settings, the CUDA path called
through the C ABI on the whole workload and checked against the float64
oracle head by head (rules in tests/parity.py):

* one online-compaction round of a Qwen3-4B-shaped model (288 heads, a cache
  of 2048 whose first 2028 keys are halved to 1014, n = 2048, a prior β on the
  already compacted half: xinfinite.net article §5, Table 3);
* the full Qwen3-4B-shaped model at 50× (288 heads, T = n = 8192, log-normal
  budgets from 8 to 1024; zhichai.net/en summary, the results table);
* a Llama-3.1-8B-shaped 60k-token context cut KV-based into chunks of 8192
  (one full chunk, t = 819, and the 2656-key last chunk, t = 266, in one
  call; xinfinite.net article §3, Table 1);
* the tensor-core recompute of the correlations against the oracle on the
  Qwen3-4B layer.

Heads whose full float64 replay would take minutes (budgets near 1000 on
8192 × 8192 features) are checked by check_head_prefix: the first 256 picks
replayed exactly, and β, residual and output against the oracle on the GPU's
own keys.  The oracle jobs run in a spawn process pool.
"""
import numpy as np
import pytest
import torch

from attention_matching_b200 import workloads as W
from tests.parity import check_heads_parallel, check_refit_kkt, shift_for, split_head

pytestmark = pytest.mark.gpu

needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def _run(heads, budgets, topk, refit, shifts, key_bias=None, varlen=False, **kw):
    import attention_matching_b200 as am
    Q = torch.stack([h.Q for h in heads]).contiguous().cuda()
    if varlen:
        K = torch.cat([h.K for h in heads]).contiguous().cuda()
        V = torch.cat([h.V for h in heads]).contiguous().cuda()
        kw["key_offsets"] = W.key_offsets_of(heads)
    else:
        K = torch.stack([h.K for h in heads]).contiguous().cuda()
        V = torch.stack([h.V for h in heads]).contiguous().cuda()
    kb = None
    if key_bias is not None:
        kb = torch.tensor(np.concatenate(key_bias) if varlen else np.stack(key_bias), dtype=torch.float32).cuda()
    out = am.compact_heads(Q, K, V, budgets, topk=topk, refit_every=refit,
                           shift=torch.tensor(shifts, dtype=torch.float32).cuda(), key_bias=kb, trace=True, **kw)
    assert all(s in (0, 8) for s in out["status"]), out["status"]
    return out


def _job(kind, out, heads, h, budget, topk, refit, shift, key_bias=None, label="", **extra):
    Q, K, V = heads[h].f64()
    kw = dict(g=split_head(out, h), Q=Q, K=K, V=V, t=budget, topk=topk, refit=refit, shift=shift,
              key_bias=None if key_bias is None else np.asarray(key_bias, np.float64), label=label)
    kw.update(extra)
    return (kind, kw)


@needs_cuda
def test_online_round_full_size_with_prior_bias():
    """288 heads, T = 2028 (the cache of 2048 less the 20 latest keys), n = 2048,
    t = 1014, k = 4, R = 2; the first 1014 keys carry a prior β (an already
    compacted block), the rest none.  Heads checked: the first, and the ones
    the GPU left with the largest and the smallest mass residual."""
    H, T, n, t = 288, 2028, 2048, 1014
    heads = [W.structured_head(7000 + h, n=n, T=T) for h in range(H)]
    rng = np.random.default_rng(7999)
    kb = [np.float32(np.concatenate([np.log(rng.uniform(1.0, 3.0, t)), np.zeros(T - t)])) for _ in range(H)]
    shifts = [shift_for(*hd.f64()[:2], key_bias=np.float64(kb[i])) for i, hd in enumerate(heads)]
    out = _run(heads, [t] * H, 4, 2, shifts, key_bias=kb)
    res = out["residual"].cpu().numpy()
    pick = sorted({0, int(np.argmax(res)), int(np.argmin(res))})
    # the GPU's own fp64 weights solve the NNLS of its own stored features
    import attention_matching_b200 as am
    f = am.features(out, n, T, 128, [t] * H, 4, 2, am.BF16)
    for h in pick:
        check_refit_kkt(out, f, h, n)
    reps = check_heads_parallel([_job("full", out, heads, h, t, 4, 2, shifts[h], kb[h], f"online head {h}")
                                 for h in pick])
    for r in reps:
        assert r["beta_maxdiff"] <= 1e-3   # output (or fit) checked in check_head


@needs_cuda
def test_qwen3_model_full_size_budget_extremes():
    """The 288-head model at 50× with log-normal budgets: the smallest budget
    (8) and a median one checked in full, the largest (1024) by the prefix
    rule; the largest head's fp64 NNLS weights also meet the optimality
    conditions on the GPU's own features."""
    import attention_matching_b200 as am
    wl = W.qwen3_4b_model()
    shifts = [shift_for(*hd.f64()[:2]) for hd in wl.heads]
    out = _run(wl.heads, wl.budgets, wl.topk, wl.refit_every, shifts)
    b = np.array(wl.budgets)
    lo, hi = int(np.argmin(b)), int(np.argmax(b))
    mid = int(np.argsort(b)[len(b) // 2])
    assert b[hi] == 1024 and b[lo] <= 8
    jobs = [_job("full", out, wl.heads, h, wl.budgets[h], 4, 2, shifts[h], label=f"model head {h}") for h in (lo, mid)]
    jobs.append(_job("prefix", out, wl.heads, hi, wl.budgets[hi], 4, 2, shifts[hi], label=f"model head {hi}",
                     prefix=256))
    for r in check_heads_parallel(jobs):
        assert r["out_rel"] <= 2e-3
    f = am.features(out, 8192, 8192, 128, wl.budgets, 4, 2, am.BF16)
    check_refit_kkt(out, f, hi, 8192)


@needs_cuda
def test_long_context_chunks_full_size():
    """A full 8192-key chunk (t = 819) and the 2656-key last chunk (t = 266)
    of a 60000-key sequence in one call (per-head key offsets), top-k 8 with a
    refit every 2 rounds, n = 8192 reference queries per chunk."""
    chunks = W.long_sequence_chunks(5000, 60000, 8192, 8192)
    heads = [chunks[3], chunks[7]]
    assert [h.T for h in heads] == [8192, 2656]
    budgets = [W.budget_for_ratio(h.T, 10.0) for h in heads]
    assert budgets == [819, 266]
    shifts = [shift_for(*hd.f64()[:2]) for hd in heads]
    out = _run(heads, budgets, 8, 2, shifts, varlen=True)
    jobs = [_job("prefix", out, heads, 0, 819, 8, 2, shifts[0], label="chunk 3", prefix=256),
            _job("full", out, heads, 1, 266, 8, 2, shifts[1], label="last chunk")]
    for r in check_heads_parallel(jobs):
        assert r["out_rel"] <= 2e-3


@needs_cuda
def test_recompute_correlation_against_the_oracle_full_size():
    """AM_CORR_RECOMPUTE (Φ recomputed on the tensor cores every pass) on
    three heads of the Qwen3-4B layer, each checked in full."""
    import attention_matching_b200 as am
    wl = W.qwen3_4b_layer(num_heads=3)
    shifts = [shift_for(*hd.f64()[:2]) for hd in wl.heads]
    out = _run(wl.heads, wl.budgets, 4, 2, shifts, corr_mode=am.CORR_RECOMPUTE)
    reps = check_heads_parallel([_job("full", out, wl.heads, h, wl.budgets[h], 4, 2, shifts[h],
                                      label=f"recompute head {h}") for h in range(3)])
    for r in reps:
        assert r["out_rel"] <= 2e-3
