"""Pins for the float64 oracle against facts fixed outside the oracle itself:
brute force on tiny inputs, closed forms, library special cases and the
invariants the pages state.  Each test names the page passage it checks.

Pages ("Fast KV Compaction via Attention Matching"): [DeepDive] zhichai.net
deep dive; [Article] xinfinite.net article; [Summary] zhichai.net/en summary;
[News] youleyou.com rewrite.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.optimize import nnls as scipy_nnls

from oracle import am_oracle as O
from attention_matching_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# Φ and m: brute-force scalar loops ([DeepDive] §1.6 definition of Φ and m)
# --------------------------------------------------------------------------

def test_mass_features_bruteforce():
    rng = np.random.default_rng(1)
    n, T, d = 5, 7, 3
    Q, K = rng.standard_normal((n, d)), rng.standard_normal((T, d))
    b = rng.standard_normal(T)
    c = 0.7
    Phi, m, c_used = O.mass_features(Q, K, shift=c, key_bias=b)
    assert c_used == c
    for i in range(n):
        tot = 0.0
        for j in range(T):
            dot = 0.0
            for k in range(d):
                dot += Q[i, k] * K[j, k]
            e = math.exp(dot / math.sqrt(d) + b[j] - c)
            assert abs(Phi[i, j] - e) <= 1e-14 * e
            tot += e
        assert abs(m[i] - tot) <= 1e-13 * tot
    # default shift is the largest logit, so max Φ is exactly 1
    Phi2, _, c2 = O.mass_features(Q, K, key_bias=b)
    assert Phi2.max() == 1.0
    assert abs(c2 - max(Q[i] @ K[j] / math.sqrt(d) + b[j] for i in range(n) for j in range(T))) < 1e-12


def test_target_outputs_match_sdpa():
    """Y = ΦV/m is ordinary softmax attention (library special case, b = 0)."""
    rng = np.random.default_rng(2)
    n, T, d = 17, 33, 8
    Q, K, V = (rng.standard_normal(s) for s in ((n, d), (T, d), (T, d)))
    Phi, m, _ = O.mass_features(Q, K)
    Y = O.target_outputs(Phi, V, m)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None])[0].numpy()
    np.testing.assert_allclose(Y, ref, rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# Mixing identity ([DeepDive] §1.3, [Article] §1)
# --------------------------------------------------------------------------

def test_mixing_identity_two_blocks():
    rng = np.random.default_rng(3)
    n, d = 11, 16
    Q = rng.standard_normal((n, d))
    K1, V1 = rng.standard_normal((9, d)), rng.standard_normal((9, d))
    K2, V2 = rng.standard_normal((14, d)), rng.standard_normal((14, d))
    full = O.attention_output(Q, np.vstack([K1, K2]), np.vstack([V1, V2]))
    o1, l1 = O.local_attention(Q, K1, V1)
    o2, l2 = O.local_attention(Q, K2, V2)
    mixed = O.mix_blocks([o1, o2], [l1, l2])
    assert np.linalg.norm(mixed - full) <= 1e-12 * np.linalg.norm(full)
    # torch's logsumexp pins the log-mass
    s1 = torch.from_numpy(Q @ K1.T / math.sqrt(d))
    np.testing.assert_allclose(l1, torch.logsumexp(s1, dim=1).numpy(), rtol=1e-13)


def test_mixing_identity_with_bias_block():
    """A compacted block carries β: its mass is Σ exp(s + β) and it mixes
    with a fresh block exactly like a plain block of keys ([DeepDive] §1.4)."""
    rng = np.random.default_rng(4)
    n, d = 7, 8
    Q = rng.standard_normal((n, d))
    Kc, Vc, beta = rng.standard_normal((5, d)), rng.standard_normal((5, d)), rng.standard_normal(5)
    Kf, Vf = rng.standard_normal((6, d)), rng.standard_normal((6, d))
    full = O.attention_output(Q, np.vstack([Kc, Kf]), np.vstack([Vc, Vf]),
                              key_bias=np.concatenate([beta, np.zeros(6)]))
    oc, lc = O.local_attention(Q, Kc, Vc, key_bias=beta)
    of, lf = O.local_attention(Q, Kf, Vf)
    assert np.linalg.norm(O.mix_blocks([oc, of], [lc, lf]) - full) <= 1e-12 * np.linalg.norm(full)
    # an integer bias log(r) is the same as r copies of the key
    r = 3
    Kdup = np.vstack([Kc[:1]] * r + [Kc[1:]])
    Vdup = np.vstack([Vc[:1]] * r + [Vc[1:]])
    b = np.zeros(5)
    b[0] = math.log(r)
    np.testing.assert_allclose(O.attention_output(Q, Kc, Vc, key_bias=b),
                               O.attention_output(Q, Kdup, Vdup), rtol=1e-12)


# --------------------------------------------------------------------------
# NNLS ([Article] §2 step 2; [News]: mass matching with C_k fixed is NNLS)
# --------------------------------------------------------------------------

def _nnls_by_enumeration(A, y):
    """Brute force: every support, unconstrained LS, keep the best feasible."""
    p = A.shape[1]
    best = (math.inf, np.zeros(p))
    for k in range(p + 1):
        for sup in itertools.combinations(range(p), k):
            x = np.zeros(p)
            if sup:
                z, *_ = np.linalg.lstsq(A[:, sup], y, rcond=None)
                if np.any(z < 0):
                    continue
                x[list(sup)] = z
            res = np.linalg.norm(A @ x - y)
            if res < best[0] - 1e-15:
                best = (res, x)
    return best[1]


@pytest.mark.parametrize("seed", range(6))
def test_nnls_matches_enumeration_and_scipy(seed):
    rng = np.random.default_rng(100 + seed)
    A = rng.standard_normal((12, 6))
    y = rng.standard_normal(12)
    x = O.nnls(A, y)
    np.testing.assert_allclose(x, _nnls_by_enumeration(A, y), atol=1e-10)
    np.testing.assert_allclose(x, scipy_nnls(A, y)[0], atol=1e-10)
    kkt = O.nnls_kkt_residual(A, y, x)
    assert kkt["min_x"] >= 0 and kkt["stationarity"] < 1e-9 and kkt["dual_feasibility"] < 1e-9


@pytest.mark.parametrize("seed", range(4))
def test_nnls_warm_start_reaches_the_same_minimiser(seed):
    """A feasible warm start (as the OMP refits use) ends where a cold start does."""
    rng = np.random.default_rng(200 + seed)
    A = rng.random((40, 12)) + 0.1 * rng.standard_normal((40, 12))
    y = rng.random(40)
    cold = O.nnls(A, y)
    for x0 in (np.zeros(12), rng.random(12), np.where(rng.random(12) < 0.5, rng.random(12), 0.0), cold):
        np.testing.assert_allclose(O.nnls(A, y, x0=x0), cold, atol=1e-10)
    np.testing.assert_allclose(cold, _nnls_by_enumeration(A, y), atol=1e-10)


@pytest.mark.parametrize("seed", range(3))
def test_nnls_reaches_the_minimiser_when_the_residual_is_tiny(seed):
    """Brute force with columns of very different mass (one sink-like column
    1e4 times the others, as attention features have): y = A[:, :5]x* + c·a_5
    lies in the cone of A, and after the 5-column fit (also the warm start an
    OMP refit begins from) a_5's gradient is ~1e-10·‖a_5‖‖y‖, far below
    1e-13·‖A‖_F·‖y‖.  The minimiser (and the enumeration) reach residual ~0;
    a stopping test on the raw gradient against ‖A‖_F·‖y‖ ends at ~1e-10·‖y‖."""
    rng = np.random.default_rng(900 + seed)
    n = 30
    A = rng.random((n, 6)) + 0.2
    A[:, 0] *= 1e4
    x_true = rng.random(5) + 0.5
    y = A[:, :5] @ x_true + 1e-5 * A[:, 5]
    best = _nnls_by_enumeration(A, y)
    rb = np.linalg.norm(A @ best - y)
    assert rb < 1e-13 * np.linalg.norm(y)
    x5 = np.linalg.lstsq(A[:, :5], y, rcond=None)[0]
    for x0 in (None, np.concatenate([x5, [0.0]])):
        x = O.nnls(A, y, x0=x0)
        ry = np.linalg.norm(A @ x - y)
        assert ry <= rb + 1e-13 * np.linalg.norm(y), (ry, rb)
        assert x[5] > 0 and x.min() >= 0


def test_nnls_single_column_closed_form():
    rng = np.random.default_rng(5)
    phi = rng.random(20)
    y = rng.random(20)
    assert abs(O.nnls(phi[:, None], y)[0] - (phi @ y) / (phi @ phi)) < 1e-14
    assert O.nnls(phi[:, None], -y)[0] == 0.0


def test_kkt_checker_flags_points_that_are_not_optimal():
    """The KKT checker that accepts the GPU's fp64 weights must reject points
    that are not minimisers.  Closed form first: with A = I and y = (1, -1)
    the minimiser is x = (1, 0) with gradient g = x - y = (0, 1); at x = 0
    the first variable has g_0 = -1 off the support (a descent direction),
    at x = (1.5, 0) it has g_0 = 0.5 on the support, and a negative entry is
    reported as min_x.  Then perturbations of scipy's minimiser of a random
    problem: scaling one positive weight, zeroing one, and making a zero one
    positive each break one condition by far more than the 1e-10 bar."""
    A = np.eye(2)
    y = np.array([1.0, -1.0])
    ok = O.nnls_kkt_residual(A, y, np.array([1.0, 0.0]))
    assert ok["min_x"] == 0.0 and ok["stationarity"] == 0.0 and ok["dual_feasibility"] == 0.0
    at0 = O.nnls_kkt_residual(A, y, np.zeros(2))
    assert abs(at0["dual_feasibility"] - 1.0 / math.sqrt(2.0)) < 1e-15
    over = O.nnls_kkt_residual(A, y, np.array([1.5, 0.0]))
    assert abs(over["stationarity"] - 0.5 / math.sqrt(2.0)) < 1e-15
    assert O.nnls_kkt_residual(A, y, np.array([1.0, -0.25]))["min_x"] == -0.25

    rng = np.random.default_rng(61)
    A = rng.random((60, 14)) + 0.05 * rng.standard_normal((60, 14))
    y = A[:, :4] @ rng.uniform(0.5, 2.0, 4) - 0.3 * A[:, 9] + 0.01 * rng.standard_normal(60)
    x = scipy_nnls(A, y)[0]
    on, off = np.flatnonzero(x > 0), np.flatnonzero(x == 0)
    assert on.size and off.size
    base = O.nnls_kkt_residual(A, y, x)
    assert base["stationarity"] < 1e-10 and base["dual_feasibility"] < 1e-10
    bad = x.copy()
    bad[on[0]] *= 1.01
    assert O.nnls_kkt_residual(A, y, bad)["stationarity"] > 1e-6
    bad = x.copy()
    bad[on[0]] = 0.0
    assert O.nnls_kkt_residual(A, y, bad)["dual_feasibility"] > 1e-6
    bad = x.copy()
    g = A.T @ (A @ x - y)
    j = off[np.argmax(g[off])]          # the zero weight whose gradient is most positive
    bad[j] = 0.1
    assert O.nnls_kkt_residual(A, y, bad)["stationarity"] > 1e-6


def test_nnls_kkt_on_exp_features():
    """Mass-fit-shaped problem (positive, correlated columns)."""
    h = W.iid_head(7, n=128, T=40, d=16, dtype="fp32")
    Q, K, _ = h.f64()
    Phi, m, _ = O.mass_features(Q, K)
    x = O.nnls(Phi, m)
    kkt = O.nnls_kkt_residual(Phi, m, x)
    assert kkt["min_x"] >= 0 and kkt["stationarity"] < 1e-9 and kkt["dual_feasibility"] < 1e-9
    np.testing.assert_allclose(x, scipy_nnls(Phi, m, maxiter=1000)[0], rtol=1e-7, atol=1e-9)


# --------------------------------------------------------------------------
# OMP ([DeepDive] §1.6; [Article] §2 Fig. 1 and §3 top-k + lazy refit)
# --------------------------------------------------------------------------

def test_omp_tiny_bruteforce_two_picks():
    """T=6, t=2, plain OMP: each step recomputed with scalar loops and
    brute-force NNLS."""
    rng = np.random.default_rng(8)
    n, T, d = 9, 6, 4
    Q, K = rng.standard_normal((n, d)), rng.standard_normal((T, d))
    Phi, m, _ = O.mass_features(Q, K)
    S, w, rounds = O.omp_select(Phi, m, 2, 1, 1)
    corr = [sum(m[i] * Phi[i, j] for i in range(n)) for j in range(T)]
    j1 = max(range(T), key=lambda j: (corr[j], -j))
    assert S[0] == j1
    w1 = max(0.0, sum(Phi[i, j1] * m[i] for i in range(n)) / sum(Phi[i, j1] ** 2 for i in range(n)))
    r = [m[i] - Phi[i, j1] * w1 for i in range(n)]
    corr2 = [sum(r[i] * Phi[i, j] for i in range(n)) if j != j1 else -math.inf for j in range(T)]
    j2 = max(range(T), key=lambda j: (corr2[j], -j))
    assert S[1] == j2
    np.testing.assert_allclose(w, _nnls_by_enumeration(Phi[:, [j1, j2]], m), rtol=1e-10)
    np.testing.assert_allclose(rounds[0]["c"], corr, rtol=1e-12)


def test_omp_full_budget_is_exact():
    """t = T: w = 1, zero mass residual; ridge = 0 gives C_v = V."""
    h = W.iid_head(9, n=64, T=12, d=8, dtype="fp32")
    Q, K, V = h.f64()
    r = O.compact_head(Q, K, V, 12, 1, 1, ridge=0.0)
    np.testing.assert_allclose(r["w"], np.ones(12), rtol=1e-9)
    assert r["residual"] < 1e-12
    np.testing.assert_allclose(r["C_v"], V, atol=1e-8)
    np.testing.assert_allclose(r["beta"], np.zeros(12), atol=1e-9)


def test_omp_exact_recovery_duplicated_keys():
    """K holds g distinct keys each repeated r times (different V per copy):
    with t = g, OMP takes one copy per group (the lowest index), w = r,
    β = log r, zero residual, and C_v is the mean of each group's values."""
    rng = np.random.default_rng(10)
    g, rep, d, n = 5, 3, 6, 40
    base = rng.standard_normal((g, d))
    order = rng.permutation(g * rep)
    K = np.repeat(base, rep, axis=0)[order]
    V = rng.standard_normal((g * rep, d))
    Q = rng.standard_normal((n, d))
    res = O.compact_head(Q, K, V, g, 1, 1, ridge=0.0)
    group = np.repeat(np.arange(g), rep)[order]
    firsts = sorted(int(np.flatnonzero(group == a)[0]) for a in range(g))
    assert list(res["indices"]) == firsts
    np.testing.assert_allclose(res["w"], np.full(g, float(rep)), rtol=1e-9)
    np.testing.assert_allclose(res["beta"], np.full(g, math.log(rep)), atol=1e-9)
    assert res["residual"] < 1e-12
    for l, j in enumerate(res["indices"]):
        np.testing.assert_allclose(res["C_v"][l], V[group == group[j]].mean(axis=0), atol=1e-8)
    O_c = O.reconstructed_output(Q, res["C_k"], res["beta"], res["C_v"])
    np.testing.assert_allclose(O_c, O.attention_output(Q, K, V), atol=1e-9)


def test_omp_shift_invariance():
    h = W.structured_head(11, n=256, T=256, d=32, rank=8)
    Q, K, V = h.f64()
    c = O.max_logit(Q, K)
    a = O.compact_head(Q, K, V, 12, 4, 2, shift=c)
    b = O.compact_head(Q, K, V, 12, 4, 2, shift=c + 3.0)
    assert list(a["indices"]) == list(b["indices"])
    np.testing.assert_allclose(a["w"], b["w"], rtol=1e-9)
    np.testing.assert_allclose(a["beta"], b["beta"], atol=1e-9)
    np.testing.assert_allclose(a["C_v"], b["C_v"], rtol=1e-8, atol=1e-10)


def test_omp_permutation_equivariance():
    h = W.iid_head(12, n=96, T=48, d=16, dtype="fp32")
    Q, K, V = h.f64()
    perm = np.random.default_rng(13).permutation(48)
    a = O.compact_head(Q, K, V, 6, 1, 1)
    b = O.compact_head(Q, K[perm], V[perm], 6, 1, 1)
    assert sorted(perm[b["indices"]].tolist()) == a["indices"].tolist()
    ia = np.argsort(a["indices"])
    ib = np.argsort(perm[b["indices"]])
    np.testing.assert_allclose(a["beta"][ia], b["beta"][ib], atol=1e-9)
    np.testing.assert_allclose(a["C_v"][ia], b["C_v"][ib], atol=1e-8)


def test_omp_lazy_refit_reading():
    """Adopted reading of top-k batching with lazy refit: R rounds of k picks
    between refits take the top k·R of one correlation vector, so (4, 2)
    selects exactly what (8, 1) does."""
    h = W.structured_head(14, n=512, T=512, d=32, rank=8)
    Q, K, V = h.f64()
    Phi, m, _ = O.mass_features(Q, K)
    S42, w42, _ = O.omp_select(Phi, m, 30, 4, 2)
    S81, w81, _ = O.omp_select(Phi, m, 30, 8, 1)
    assert S42 == S81
    np.testing.assert_allclose(w42, w81, rtol=1e-12)


def test_best_subset_sixteen_keys_known_optimum():
    """Exhaustive search over T = 16 keys on a problem whose optimum is known
    by construction: m is an exact positive combination of three columns of a
    positive Φ, so that subset fits with zero residual while no other subset
    of three generic columns can.  The search must return it, and its
    residual must equal the minimum over all subsets computed independently
    with scipy's NNLS; OMP's residual is never below it."""
    rng = np.random.default_rng(77)
    n, T, t = 40, 16, 3
    Phi = rng.uniform(0.05, 1.0, (n, T))
    S_true = [2, 9, 13]
    m = Phi[:, S_true] @ np.array([0.7, 1.9, 0.4])
    res, S = O.best_subset(Phi, m, t)
    assert S == S_true and res < 1e-12
    indep = min(np.linalg.norm(m - Phi[:, list(c)] @ scipy_nnls(Phi[:, list(c)], m)[0])
                for c in itertools.combinations(range(T), t)) / np.linalg.norm(m)
    assert abs(res - indep) < 1e-12
    for k in (1, 2):
        res_k, S_k = O.best_subset(Phi, m, k)
        indep_k = min(np.linalg.norm(m - Phi[:, list(c)] @ scipy_nnls(Phi[:, list(c)], m)[0])
                      for c in itertools.combinations(range(T), k)) / np.linalg.norm(m)
        assert abs(res_k - indep_k) < 1e-12
        Somp, w, _ = O.omp_select(Phi, m, k, 1, 1)
        assert res_k <= O.mass_residual(Phi, m, Somp, w) + 1e-12


def test_omp_greedy_never_beats_best_subset():
    """Exhaustive best-subset NNLS on T ≤ 10: its residual is ≤ OMP's, and
    for t = 1 plain OMP's first pick has positive correlation."""
    for seed in range(4):
        h = W.iid_head(20 + seed, n=32, T=10, d=4, dtype="fp32")
        Q, K, _ = h.f64()
        Phi, m, _ = O.mass_features(Q, K)
        for t in (1, 2, 3):
            S, w, _ = O.omp_select(Phi, m, t, 1, 1)
            best, _ = O.best_subset(Phi, m, t)
            assert best <= O.mass_residual(Phi, m, S, w) + 1e-12


def test_omp_budget_bounds():
    Phi = np.ones((3, 4))
    with pytest.raises(ValueError):
        O.omp_select(Phi, Phi.sum(1), 0)
    with pytest.raises(ValueError):
        O.omp_select(Phi, Phi.sum(1), 5)


# --------------------------------------------------------------------------
# β, design matrix and value fit ([DeepDive] §1.6 β = log w; [Article] §2
# step 3 OLS; [News] OLS for C_v with C_k and β fixed)
# --------------------------------------------------------------------------

def test_bias_floor_and_prior():
    beta, w_eff = O.bias_from_weights(np.array([2.0, 0.0, 0.5]), np.array([0.1, 0.2, 0.3]), 1e-12)
    np.testing.assert_allclose(w_eff, [2.0, 2e-12, 0.5])
    np.testing.assert_allclose(beta, [math.log(2) + 0.1, math.log(2e-12) + 0.2, math.log(0.5) + 0.3])


def test_design_matrix_is_compact_softmax():
    rng = np.random.default_rng(15)
    n, T, d = 20, 30, 8
    Q, K = rng.standard_normal((n, d)), rng.standard_normal((T, d))
    Phi, m, c = O.mass_features(Q, K)
    idx = [2, 5, 11, 29]
    w = rng.random(4) + 0.1
    A = O.design_matrix(Phi[:, idx], w)
    s = torch.from_numpy(Q @ K[idx].T / math.sqrt(d) + np.log(w))
    np.testing.assert_allclose(A, torch.softmax(s, dim=1).numpy(), rtol=1e-12)


def test_value_fit_orthogonality_and_lstsq():
    rng = np.random.default_rng(16)
    A = rng.random((50, 7))
    A /= A.sum(1, keepdims=True)
    Y = rng.standard_normal((50, 5))
    C0, lam0 = O.value_fit(A, Y, ridge=0.0)
    assert lam0 == 0.0
    assert np.linalg.norm(A.T @ (Y - A @ C0)) <= 1e-10 * np.linalg.norm(A) * np.linalg.norm(Y)
    np.testing.assert_allclose(C0, np.linalg.lstsq(A, Y, rcond=None)[0], rtol=1e-9, atol=1e-10)
    C1, lam1 = O.value_fit(A, Y, ridge=1e-6)
    assert abs(lam1 - 1e-6 * np.trace(A.T @ A) / 7) < 1e-20
    np.testing.assert_allclose(A.T @ (Y - A @ C1), lam1 * C1, atol=1e-12)
    np.testing.assert_allclose(C1, np.linalg.solve(A.T @ A + lam1 * np.eye(7), A.T @ Y), rtol=1e-8)


# --------------------------------------------------------------------------
# Highest-attention selection ([Summary] "Method Family": AM-Highest)
# --------------------------------------------------------------------------

def test_highest_attention_select():
    rng = np.random.default_rng(17)
    n, T, d = 16, 24, 8
    Q, K = rng.standard_normal((n, d)), rng.standard_normal((T, d))
    score = torch.softmax(torch.from_numpy(Q @ K.T / math.sqrt(d)), dim=1).sum(0).numpy()
    sel = O.highest_attention_select(Q, K, 5)
    assert sorted(sel) == sorted(np.argsort(-score, kind="stable")[:5].tolist())
    assert sel == np.argsort(-score, kind="stable")[:5].tolist()      # pick order: largest first
    # with a prior per-key bias, the softmax takes it as an additive logit term
    b = rng.standard_normal(T)
    score_b = torch.softmax(torch.from_numpy(Q @ K.T / math.sqrt(d) + b[None, :]), dim=1).sum(0).numpy()
    assert O.highest_attention_select(Q, K, 7, key_bias=b) == np.argsort(-score_b, kind="stable")[:7].tolist()
    # exact ties go to the lower key: duplicated keys share a score
    K2 = np.concatenate([K[:3], K[:3]])
    sel2 = O.highest_attention_select(Q, K2, 6)
    for j in range(3):
        assert sel2.index(j) < sel2.index(j + 3)


# --------------------------------------------------------------------------
# Facts the pages print
# --------------------------------------------------------------------------

def test_golden_page_facts():
    with open(os.path.join(GOLDEN, "page_facts.json")) as f:
        facts = json.load(f)
    # per compacted token the cache stores one key row, one value row and one
    # scalar β: (2d+1)/(2d) of a plain token's storage ([DeepDive] §1.4)
    for d in (64, 128):
        assert (2 * d + 1) / (2 * d) == pytest.approx(eval(facts["bias_memory_overhead"], {"d": d}))
    # online compaction keeps the latest 20 tokens and halves the rest
    # ([Article] §5, Table 3 context)
    assert facts["online_keep_latest"] == 20 and facts["online_ratio"] == 0.5


# --------------------------------------------------------------------------
# Workload generator invariants (input recipe, not oracle arithmetic)
# --------------------------------------------------------------------------

def test_lognormal_budget_schedule():
    b = W.lognormal_budgets(4999, 288, 47186)
    assert sum(b) == 47186 and min(b) >= 4 and max(b) <= 1024 and len(b) == 288
    assert W.budget_for_ratio(8192, 50) == 164
    assert W.budget_for_ratio(2028, 2) == 1014


def test_structured_head_is_deterministic_bf16():
    a = W.structured_head(3, n=64, T=128)
    b = W.structured_head(3, n=64, T=128)
    assert a.K.dtype == torch.bfloat16 and torch.equal(a.K, b.K) and torch.equal(a.Q, b.Q)
