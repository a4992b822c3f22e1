"""Device-side failure paths, each returning a status through the C ABI
without faulting, trapping or hanging the GPU: non-finite inputs, the NNLS
iteration cap, a bounded wait that runs out, and reference queries whose
fp32 features all underflow.  Per-head statuses are read with
am_get_status (tests/parity.py rules for the heads that must stay exact)."""
import numpy as np
import pytest
import torch

from attention_matching_b200 import workloads as W
from oracle import am_oracle as O
from tests.parity import check_head, shift_for, split_head

pytestmark = pytest.mark.gpu

needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def _stack(heads):
    return [torch.stack([getattr(h, a) for h in heads]).contiguous().cuda() for a in ("Q", "K", "V")]


@needs_cuda
def test_nonfinite_inputs_flag_their_heads_only():
    """A NaN key in head 1 and an infinite query in head 2 give those heads
    AM_ERR_NONFINITE; head 0, in the same call, still matches the oracle."""
    import attention_matching_b200 as am
    heads = [W.structured_head(640 + h, n=256, T=300) for h in range(3)]
    Q, K, V = _stack(heads)
    K[1, 17, 5] = float("nan")
    Q[2, 3, 0] = float("inf")
    shift0 = shift_for(*heads[0].f64()[:2])
    out = am.compact_heads(Q, K, V, [12, 12, 12], topk=4, refit_every=2, trace=True, check=False)
    status, worst = am.get_status(out["workspace"], 3)
    assert status[1] == 4 and status[2] == 4 and worst == 4, status
    assert status[0] == 0, status
    Qf, Kf, Vf = heads[0].f64()
    g = split_head(out, 0)
    assert abs(float(out["shift"][0]) - shift0) <= 1e-5 * abs(shift0)
    check_head(g, Qf, Kf, Vf, 12, 4, 2, float(out["shift"][0]), label="finite head beside non-finite ones")
    with pytest.raises(am.AmError) as e:
        am.compact_heads(Q, K, V, [12, 12, 12], topk=4, refit_every=2)
    assert e.value.code == 4


@needs_cuda
def test_nnls_iteration_cap_is_a_warning():
    """nnls_max_iter = 1: refits that need more active-set steps stop at the
    cap and report AM_WARN_NOT_CONVERGED; the call still completes, with
    finite outputs, and a warning does not raise in the binding."""
    import attention_matching_b200 as am
    heads = [W.twin_keys_head(650 + h, n=384, T=400) for h in range(3)]
    Q, K, V = _stack(heads)
    out = am.compact_heads(Q, K, V, [60, 60, 60], topk=4, refit_every=2, nnls_max_iter=1)
    assert set(out["status"]) <= {0, 8} and 8 in out["status"], out["status"]
    for k in ("beta", "C_v"):
        assert torch.isfinite(out[k]).all(), k
    full = am.compact_heads(Q, K, V, [60, 60, 60], topk=4, refit_every=2)
    assert full["status"] == [0, 0, 0], full["status"]


@needs_cuda
def test_wait_budget_runs_out_then_the_next_call_is_exact():
    """A wait budget of one clock cycle: the tensor-core feature pass's first
    waits run out, every head records AM_ERR_TIMEOUT, and the kernel drains
    what it issued and releases its tensor memory.  The next call on the same
    workspace, with the default budget, gives the result of a fresh call bit
    for bit."""
    import attention_matching_b200 as am
    heads = [W.structured_head(660 + h, n=640, T=700) for h in range(2)]
    Q, K, V = _stack(heads)
    shifts = torch.tensor([shift_for(*h.f64()[:2]) for h in heads], dtype=torch.float32).cuda()
    ref = am.compact_heads(Q, K, V, [20, 33], topk=4, refit_every=2, shift=shifts)
    ws = torch.zeros_like(ref["workspace"])
    bad = am.compact_heads(Q, K, V, [20, 33], topk=4, refit_every=2, shift=shifts, workspace=ws, wait_cycles=1,
                           check=False)
    status, worst = am.get_status(bad["workspace"], 2)
    assert status == [6, 6] and worst == 6, status
    good = am.compact_heads(Q, K, V, [20, 33], topk=4, refit_every=2, shift=shifts, workspace=ws)
    assert good["status"] == [0, 0]
    for k in ("indices", "C_k", "beta", "C_v"):
        assert torch.equal(good[k], ref[k]), k


@needs_cuda
def test_mass_underflow_is_reported_per_head():
    """Reference queries that mix a sink key in reach logits near 130, so the
    head's shift (its largest logit) leaves almost every other query with all
    fp32 features below the smallest normal number.  That head reports
    AM_WARN_MASS_UNDERFLOW (its zero-mass queries drop out of the fits); a
    head of ordinary queries in the same call reports nothing and matches the
    oracle."""
    import attention_matching_b200 as am
    heads = [W.structured_head(620, n=512, T=600, sink_queries=True), W.structured_head(630, n=512, T=600)]
    # the float64 logits say which queries underflow: best logit below the shift by more than 87.3
    s0 = O.logits(*heads[0].f64()[:2])
    assert ((s0.max(axis=1) - s0.max()) * np.log2(np.e) < -127).sum() > 100
    s1 = O.logits(*heads[1].f64()[:2])
    assert (s1.max(axis=1) - s1.max()).min() > -40
    Q, K, V = _stack(heads)
    out = am.compact_heads(Q, K, V, [16, 16], topk=4, refit_every=2, trace=True)
    assert out["status"] == [10, 0], out["status"]
    Qf, Kf, Vf = heads[1].f64()
    check_head(split_head(out, 1), Qf, Kf, Vf, 16, 4, 2, float(out["shift"][1]), label="ordinary head")
