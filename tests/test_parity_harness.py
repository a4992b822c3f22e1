"""CPU checks of the GPU acceptance harness itself (tests/parity.py): fed the
oracle's own compaction it must pass, and it must fail on planted mistakes
(a wrong β, a swapped pick, a wrong value row).  Small heads only."""
import numpy as np
import pytest

from attention_matching_b200 import workloads as W
from oracle import am_oracle as O
from tests.parity import check_head, check_head_prefix, shift_for


def _as_gpu(o):
    """The oracle's result in the shape split_head gives a GPU result."""
    return {"indices": o["indices"].copy(), "C_k": o["C_k"].copy(), "beta": o["beta"].copy(),
            "C_v": o["C_v"].copy(), "pick_order": list(o["pick_order"]), "w": o["w"].copy()}


@pytest.fixture(scope="module")
def head():
    h = W.structured_head(610, n=300, T=400)
    Q, K, V = h.f64()
    c = shift_for(Q, K)
    return Q, K, V, c, O.compact_head(Q, K, V, 48, 4, 2, shift=c)


def test_harness_accepts_the_oracle(head):
    Q, K, V, c, o = head
    rep = check_head(_as_gpu(o), Q, K, V, 48, 4, 2, c)
    assert rep["same_set"] and rep["beta_maxdiff"] < 1e-9 and rep["out_rel"] < 1e-9
    rep = check_head_prefix(_as_gpu(o), Q, K, V, 48, 4, 2, c, prefix=16)
    assert rep["beta_maxdiff"] < 1e-9 and rep["out_rel"] < 1e-9


@pytest.mark.parametrize("check", ["full", "prefix"])
def test_harness_rejects_planted_mistakes(head, check):
    Q, K, V, c, o = head
    run = (lambda g: check_head(g, Q, K, V, 48, 4, 2, c)) if check == "full" else \
          (lambda g: check_head_prefix(g, Q, K, V, 48, 4, 2, c, prefix=16))
    g = _as_gpu(o)
    g["beta"][np.argmax(o["w"])] += 5e-3                     # one β off by more than 1e-3
    with pytest.raises(AssertionError):
        run(g)
    g = _as_gpu(o)
    g["C_v"][0] += 0.5 * np.abs(g["C_v"]).max()               # one value row moved
    with pytest.raises(AssertionError):
        run(g)
    g = _as_gpu(o)
    # an early pick replaced by the unselected key with the lowest first-round correlation
    c0 = o["rounds"][0]["c"]
    free = [j for j in np.argsort(c0) if j not in set(o["pick_order"])]
    g["pick_order"][1] = int(free[0])
    g["indices"] = np.sort(np.asarray(g["pick_order"]))
    g["C_k"] = K[g["indices"]]
    with pytest.raises(AssertionError):
        run(g)


def test_undetermined_weights_flags_only_ill_posed_splits():
    """On well-separated columns every weight is fixed by the data; when a
    column is repeated with a relative jitter far below fp32 precision the
    split of weight between the twins is not, and only those twins are
    flagged."""
    from tests.parity import undetermined_weights
    rng = np.random.default_rng(71)
    A = rng.uniform(0.1, 1.0, (200, 6))
    y = A @ np.array([1.0, 0.5, 2.0, 0.7, 1.3, 0.9])
    w = O.nnls(A, y)
    assert not undetermined_weights(A, y, w).any()
    B = np.concatenate([A, A[:, :1] * (1.0 + 1e-9 * rng.standard_normal((200, 1)))], axis=1)
    wb = O.nnls(B, y)
    flags = undetermined_weights(B, y, wb)
    assert set(np.flatnonzero(flags)) <= {0, 6}
