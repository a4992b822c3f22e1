"""The synthetic workloads' recipes on CPU: the long-context chunking and its
budgets, the online rounds' cache arithmetic, and the full model's budget
schedule, as the bench and the full-size tests use them."""
import numpy as np

from attention_matching_b200 import workloads as W


def test_long_context_sequence_chunks_budgets_and_offsets():
    wl = W.llama31_8b_longctx(max_sequences=1)
    heads = wl.heads
    assert [h.T for h in heads] == [8192] * 7 + [2656]          # 60000 keys, KV-based chunks
    assert wl.budgets == [819] * 7 + [266]                      # round-half-up(T / 10)
    assert wl.topk == 8 and wl.refit_every == 2
    offs = list(wl.key_offsets)
    assert offs == [0] + list(np.cumsum([h.T for h in heads]))  # packed end to end
    for h in heads:
        assert tuple(h.Q.shape) == (8192, 128) and tuple(h.K.shape) == (h.T, 128) and h.V.shape == h.K.shape
        assert str(h.Q.dtype) == "torch.bfloat16"
    # sinks only at global positions 0-3, so only in chunk 0
    norms0 = heads[0].K.float().norm(dim=1)
    assert float(norms0[:4].min()) > 2.5 * float(norms0[4:].median())
    norms1 = heads[1].K.float().norm(dim=1)
    assert float(norms1[:4].max()) < 2.5 * float(norms1[4:].median())
    # consecutive chunks are slices of one sequence: a different seed gives a different sequence
    other = W.llama31_8b_longctx(max_sequences=1, seed_base=5001).heads[0]
    assert not bool((other.K[:16] == heads[0].K[:16]).all())


def test_online_round_cache_arithmetic():
    on = W.OnlineHeads(2, seed=3000)
    assert on.compact_len == 2028 and on.budget == 1014          # keep the latest 20, halve the rest
    heads = on.next_round(None)
    # the compaction input is the cache minus the latest 20 keys (kept as they are);
    # the reference queries are drawn against the whole 2048-key cache
    assert [h.T for h in heads] == [2028, 2028] and tuple(heads[0].Q.shape) == (2048, 128)
    assert heads[0].key_bias is not None and not np.any(heads[0].key_bias)   # round 1: no prior bias


def test_model_budget_schedule():
    b = W.lognormal_budgets(4999, 288, 47186)
    assert len(b) == 288 and sum(b) == 47186 and min(b) == 8 and max(b) == 1024
    assert b == W.lognormal_budgets(4999, 288, 47186)            # seeded
