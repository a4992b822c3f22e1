"""Float64 CPU oracle for Attention-Matching KV compaction (AM-OMP).

TEST INFRASTRUCTURE ONLY.  This module is the independent, slow, plain
restatement of what the compaction path computes.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py`` (its ``cpu_baseline`` leg and its
``--impl reference`` arm) may import it.  The library in
``attention_matching_b200`` never imports it and shares no code with it.

Sources (pages on "Fast KV Compaction via Attention Matching", cited by
title and section):

* [DeepDive] zhichai.net, "MIT AM-OMP：Fast KV Compaction via Attention
  Matching 完整技术解析": §1.3 mixing identity and attention mass, §1.4 scalar
  bias, §1.6 the OMP key-selection loop and β = log w.
* [Article] xinfinite.net, "大模型上下文卡壳？MIT 用线性回归轻松破局": §1 mixing
  identity, §2 the three steps (step 2: key selection + NNLS bias fit, Fig. 1
  and Fig. 2; step 3: value fit by ordinary least squares), §3 top-k batched
  selection with lazy refit (Table 1).
* [Summary] zhichai.net/en, "MIT AM-OMP: Fast KV Compaction via Attention
  Matching — Full Technical Analysis": "Key Points" (mass definition),
  "The Three-Step Closed-Form Pipeline", "Method Family and Trade-offs".
* [News] youleyou.com, "MIT注意力匹配：内存暴降50倍精度无损…": the two matching
  conditions (their Eq. 1 and 2, named but not printed), NNLS for β with C_k
  fixed, OLS for C_v, and the "highest attention keys" selector.

Readings where the pages are silent or garbled (each is listed with its
reason in the design notes of this repository):

* logits carry the usual 1/√d scale (the pages print exp(q·k) without it);
* Φ uses one per-head scalar shift c: Φ_ij = exp(s_ij − c); every result is
  invariant to c (the NNLS minimiser scales by e^c, picks and A do not move);
* correlations are unnormalised, c_j = Σ_i r_i Φ_ij, as printed; the budget is
  always filled (no early stop on non-positive correlation); ties go to the
  lowest key index;
* top-k batching with lazy refit: each round appends the kk = min(k, t−|S|)
  best unselected keys; NNLS (and hence r) is refreshed only on every R-th
  round and on the last one;
* zero NNLS weights get the floor w_floor_rel·max(w) before the log;
* C_v solves the ridge normal equations (AᵀA + λI)C_v = AᵀY with
  λ = ridge·tr(AᵀA)/t (ridge = 1e-6); ridge = 0 gives the plain least-squares
  solution by QR;
* a prior per-key bias b (an already compacted block) enters the logits, and
  the new bias is b_S + log w.

Parity pins for every function here live in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np
from scipy.linalg import solve_triangular

F64 = np.float64


# ---------------------------------------------------------------------------
# Attention mass and the mixing identity  ([DeepDive] §1.3, [Article] §1)
# ---------------------------------------------------------------------------

def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


def logits(Q, K, scale: Optional[float] = None, key_bias=None) -> np.ndarray:
    """s_ij = (q_i · k_j)·scale + b_j, float64 [n, T]."""
    Q = np.asarray(Q, F64)
    K = np.asarray(K, F64)
    if scale is None:
        scale = default_scale(Q.shape[1])
    s = (Q @ K.T) * scale
    if key_bias is not None:
        s = s + np.asarray(key_bias, F64)[None, :]
    return s


def local_attention(Q, K, V, scale=None, key_bias=None):
    """Local attention output o_i and log-mass log Σ_j exp(s_ij) of one block."""
    s = logits(Q, K, scale, key_bias)
    mx = s.max(axis=1, keepdims=True)
    p = np.exp(s - mx)
    z = p.sum(axis=1, keepdims=True)
    o = (p @ np.asarray(V, F64)) / z
    return o, (np.log(z) + mx)[:, 0]


def attention_output(Q, K, V, scale=None, key_bias=None) -> np.ndarray:
    """softmax(Q Kᵀ·scale + b) V in float64."""
    return local_attention(Q, K, V, scale, key_bias)[0]


def mix_blocks(outputs: Sequence[np.ndarray], log_masses: Sequence[np.ndarray]) -> np.ndarray:
    """Mixing identity: attention over concatenated blocks equals the
    mass-weighted mixture Σ_b M_b o_b / Σ_b M_b of the local outputs."""
    L = np.stack(log_masses, axis=0)           # [B, n]
    mx = L.max(axis=0)
    wts = np.exp(L - mx)                        # M_b / max M
    num = sum(wts[b][:, None] * outputs[b] for b in range(len(outputs)))
    return num / wts.sum(axis=0)[:, None]


# ---------------------------------------------------------------------------
# Mass features  ([DeepDive] §1.6 "Φ_ij = exp(q_i·k_j), m_i = Σ_j Φ_ij")
# ---------------------------------------------------------------------------

def max_logit(Q, K, scale=None, key_bias=None) -> float:
    """The natural shift c = max_ij s_ij."""
    return float(logits(Q, K, scale, key_bias).max())


def mass_features(Q, K, shift: Optional[float] = None, scale=None, key_bias=None):
    """Φ = exp(s − c) [n, T] and m = Φ·1 [n]; c defaults to max_ij s_ij."""
    s = logits(Q, K, scale, key_bias)
    c = float(s.max()) if shift is None else float(shift)
    Phi = np.exp(s - c)
    return Phi, Phi.sum(axis=1), c


# ---------------------------------------------------------------------------
# Non-negative least squares  ([Article] §2 step 2, [News]: with C_k fixed
# the mass match is an NNLS problem).  Lawson-Hanson active set; the
# least-squares subproblems use Householder QR on the passive columns.
# ---------------------------------------------------------------------------

def _ls_qr(A: np.ndarray, y: np.ndarray) -> np.ndarray:
    Qm, R = np.linalg.qr(A, mode="reduced")
    return solve_triangular(R, Qm.T @ y, lower=False)


def nnls(A, y, tol: Optional[float] = None, max_iter: Optional[int] = None,
         x0: Optional[np.ndarray] = None) -> np.ndarray:
    """argmin_{x ≥ 0} ‖A x − y‖₂ by the Lawson-Hanson active-set method.

    Outer loop: move the zero variable with the largest positive scaled
    gradient g_j / ‖a_j‖, g = Aᵀ(y − Ax), into the passive set.  Inner loop:
    solve the unconstrained least squares on the passive set; if some passive
    value is not positive, step from x toward it until the first one hits
    zero, drop the zeros and resolve.  Stops when no zero variable has
    g_j > tol·‖a_j‖·‖y‖ (tol relative, default 1e-12).  The test is per
    column and relative: an absolute threshold on g stops short of the
    minimiser once ‖y − Ax‖ ≪ ‖y‖, where a variable with a tiny gradient can
    still lower the residual by a large fraction when its column is nearly
    dependent on the passive ones.

    ``x0`` (optional, feasible) starts the method from that point with its
    support as the passive set instead of from zero; the minimiser reached is
    the same.
    """
    A = np.asarray(A, F64)
    y = np.asarray(y, F64)
    nrow, p = A.shape
    if tol is None:
        tol = 1e-12
    col = np.linalg.norm(A, axis=0)
    thr = tol * col * np.linalg.norm(y)     # per-column threshold on g_j
    col = np.where(col > 0, col, 1.0)
    if max_iter is None:
        max_iter = 3 * p + 50
    x = np.zeros(p)
    passive = np.zeros(p, dtype=bool)
    blocked = np.zeros(p, dtype=bool)
    it = 0
    j = -1
    if x0 is not None:
        x = np.maximum(np.asarray(x0, F64), 0.0)
        passive = x > 0
    first = x0 is not None and passive.any()
    g = A.T @ (y - A @ x)
    while True:
        if first:
            first = False     # a warm start begins with the inner loop on its support
        else:
            cand = (~passive) & (~blocked) & (g > thr)
            if not cand.any():
                break
            idx = np.flatnonzero(cand)
            j = int(idx[np.argmax(g[idx] / col[idx])])   # argmax returns the lowest index on ties
            passive[j] = True
        while True:
            it += 1
            if it > max_iter:
                raise RuntimeError("nnls: iteration limit")
            P = np.flatnonzero(passive)
            z = np.zeros(p)
            z[P] = _ls_qr(A[:, P], y)
            if np.all(z[P] > 0):
                x = z
                break
            neg = P[z[P] <= 0]
            den = x[neg] - z[neg]
            ratios = np.where(den > 0, x[neg] / np.where(den > 0, den, 1.0), 0.0)
            k = int(np.argmin(ratios))
            x = x + ratios[k] * (z - x)
            x[neg[k]] = 0.0
            passive &= ~(passive & (x <= 0))
            x[~passive] = 0.0
        if j < 0 or passive[j]:
            blocked[:] = False
        else:
            # round-off kept the entering variable from growing: leave it out
            # until some other variable changes the active set
            blocked[j] = True
        g = A.T @ (y - A @ x)
    return x


def nnls_kkt_residual(A, y, x) -> Dict[str, float]:
    """KKT check of an NNLS solution: x ≥ 0, g = Aᵀ(Ax − y) is ≈ 0 on the
    support and ≥ 0 off it.  Returns the worst violations, each relative to
    ‖a_l‖·‖y‖ of the column concerned."""
    A = np.asarray(A, F64)
    y = np.asarray(y, F64)
    g = A.T @ (A @ x - y)
    sc = np.linalg.norm(A, axis=0) * np.linalg.norm(y)
    sc[sc == 0] = 1.0
    on = x > 0
    return {
        "min_x": float(x.min()) if x.size else 0.0,
        "stationarity": float(np.max(np.abs(g[on]) / sc[on])) if on.any() else 0.0,
        "dual_feasibility": float(np.max(np.maximum(0.0, -g[~on]) / sc[~on])) if (~on).any() else 0.0,
    }


# ---------------------------------------------------------------------------
# OMP key selection  ([DeepDive] §1.6; [Article] §2 Fig. 1; [Summary]
# "Three-Step Closed-Form Pipeline" step 1; top-k batching with lazy refit:
# [Article] §3 and Table 1)
# ---------------------------------------------------------------------------

def omp_select(Phi, m, t: int, topk: int = 1, refit_every: int = 1,
               forced_picks: Optional[Sequence[int]] = None):
    """Greedy selection of t columns of Φ to fit m with non-negative weights.

    r = m, S = [] ; each round: c = Φᵀ r, append the kk = min(k, t−|S|)
    unselected keys with the largest c (ties → lowest index); on every R-th
    round and on the last one refit w = NNLS(Φ_S, m) and r = m − Φ_S w.

    ``forced_picks`` (teacher forcing) appends those keys instead of the
    oracle's own, while still recording the oracle's view of every round.
    Returns (S in pick order, w aligned with S, per-round records).
    """
    Phi = np.asarray(Phi, F64)
    m = np.asarray(m, F64)
    n, T = Phi.shape
    if not 1 <= t <= T:
        raise ValueError("budget must satisfy 1 <= t <= T")
    S: List[int] = []
    selected = np.zeros(T, dtype=bool)
    w = np.zeros(0)
    r = m.copy()
    rnd = 0
    rounds = []
    while len(S) < t:
        c = Phi.T @ r
        kk = min(topk, t - len(S))
        cand = np.flatnonzero(~selected)
        order = cand[np.lexsort((cand, -c[cand]))]
        own = [int(j) for j in order[:kk]]
        rec = {
            "round": rnd, "kk": kk, "c": c, "own": own, "r_norm": float(np.linalg.norm(r)),
            "c_max": float(c[order[0]]),
            "c_kth": float(c[order[kk - 1]]),
            "c_next": float(c[order[kk]]) if order.size > kk else None,
        }
        if forced_picks is None:
            picks = own
        else:
            picks = [int(j) for j in forced_picks[len(S):len(S) + kk]]
            if len(set(picks)) != kk or selected[picks].any():
                raise ValueError("forced picks repeat a key")
        rec["picks"] = picks
        S.extend(picks)
        selected[picks] = True
        rnd += 1
        if rnd % refit_every == 0 or len(S) == t:
            # NNLS of the enlarged problem, started from the previous weights
            w = nnls(Phi[:, S], m, x0=np.concatenate([w, np.zeros(len(S) - w.size)]))
            r = m - Phi[:, S] @ w
            rec["refit"] = True
        else:
            rec["refit"] = False
        rounds.append(rec)
    return S, w, rounds


def mass_residual(Phi, m, S, w) -> float:
    """‖m − Φ_S w‖ / ‖m‖."""
    Phi = np.asarray(Phi, F64)
    m = np.asarray(m, F64)
    return float(np.linalg.norm(m - Phi[:, list(S)] @ np.asarray(w, F64)) / np.linalg.norm(m))


def best_subset(Phi, m, t: int):
    """Exhaustive search over every size-t column subset (tiny T only):
    returns (best residual, best subset)."""
    import itertools
    Phi = np.asarray(Phi, F64)
    T = Phi.shape[1]
    best = (math.inf, None)
    for sub in itertools.combinations(range(T), t):
        w = nnls(Phi[:, list(sub)], m)
        res = mass_residual(Phi, m, sub, w)
        if res < best[0]:
            best = (res, list(sub))
    return best


# ---------------------------------------------------------------------------
# Bias, target outputs, design matrix and value fit  ([DeepDive] §1.6
# "β = log(w)"; [Article] §2 step 3; [News] OLS for C_v with C_k, β fixed)
# ---------------------------------------------------------------------------

def bias_from_weights(w, prior_bias_S=None, floor_rel: float = 1e-12):
    """β = b_S + log max(w, floor_rel·max(w)); also returns the floored weights."""
    w = np.asarray(w, F64)
    wmax = float(w.max()) if w.size else 0.0
    w_eff = np.maximum(w, floor_rel * wmax) if wmax > 0 else np.full_like(w, floor_rel)
    beta = np.log(w_eff)
    if prior_bias_S is not None:
        beta = beta + np.asarray(prior_bias_S, F64)
    return beta, w_eff


def target_outputs(Phi, V, m) -> np.ndarray:
    """Y_i = Σ_j Φ_ij V_j / m_i — the original local attention output."""
    return (np.asarray(Phi, F64) @ np.asarray(V, F64)) / np.asarray(m, F64)[:, None]


def design_matrix(Phi_S, w_eff) -> np.ndarray:
    """A_il = Φ_{i,S_l} w_l / Σ_l' Φ_{i,S_l'} w_l' = softmax(Q C_kᵀ·scale + β)_il."""
    P = np.asarray(Phi_S, F64) * np.asarray(w_eff, F64)[None, :]
    return P / P.sum(axis=1, keepdims=True)


def cholesky_solve(G, B) -> np.ndarray:
    L = np.linalg.cholesky(G)
    Z = solve_triangular(L, B, lower=True)
    return solve_triangular(L.T, Z, lower=False)


def value_fit(A, Y, ridge: float = 1e-6):
    """C_v = argmin ‖A C_v − Y‖² (+ λ‖C_v‖²), λ = ridge·tr(AᵀA)/t.
    ridge > 0: Cholesky of AᵀA + λI; ridge = 0: least squares by QR."""
    A = np.asarray(A, F64)
    Y = np.asarray(Y, F64)
    t = A.shape[1]
    if ridge == 0.0:
        return _ls_qr(A, Y), 0.0
    G = A.T @ A
    lam = ridge * float(np.trace(G)) / t
    return cholesky_solve(G + lam * np.eye(t), A.T @ Y), lam


# ---------------------------------------------------------------------------
# The whole per-head path
# ---------------------------------------------------------------------------

def compact_head(Q, K, V, t: int, topk: int = 1, refit_every: int = 1,
                 shift: Optional[float] = None, scale: Optional[float] = None,
                 key_bias=None, ridge: float = 1e-6, floor_rel: float = 1e-12,
                 forced_picks: Optional[Sequence[int]] = None) -> Dict:
    """Φ → OMP (+NNLS) → β → C_v for one head, all float64.

    Outputs follow ascending original key position: ``indices``, ``C_k`` =
    K[indices], ``beta``, ``C_v``, ``w``; ``pick_order`` keeps the greedy
    order and ``rounds`` the per-round correlation records.
    """
    Q = np.asarray(Q, F64)
    K = np.asarray(K, F64)
    V = np.asarray(V, F64)
    Phi, m, c = mass_features(Q, K, shift, scale, key_bias)
    S, w, rounds = omp_select(Phi, m, t, topk, refit_every, forced_picks)
    order = np.argsort(S, kind="stable")
    idx = np.asarray(S, dtype=np.int64)[order]
    w_sorted = w[order]
    prior = None if key_bias is None else np.asarray(key_bias, F64)[idx]
    beta, w_eff = bias_from_weights(w_sorted, prior, floor_rel)
    Y = target_outputs(Phi, V, m)
    A = design_matrix(Phi[:, idx], w_eff)
    C_v, lam = value_fit(A, Y, ridge)
    return {
        "indices": idx, "pick_order": list(S), "w": w_sorted, "w_eff": w_eff,
        "beta": beta, "C_k": K[idx], "C_v": C_v, "shift": c,
        "residual": mass_residual(Phi, m, idx, w_sorted),
        "m": m, "Y": Y, "A": A, "lam": lam, "rounds": rounds,
    }


def reconstructed_output(Q, C_k, beta, C_v, scale=None) -> np.ndarray:
    """O = softmax(Q C_kᵀ·scale + β) C_v in float64 (the compact block's output)."""
    return attention_output(Q, C_k, C_v, scale, beta)


# ---------------------------------------------------------------------------
# Highest-attention key selection ([Summary] "Method Family": AM-Highest;
# [News] "highest attention keys").  Aggregation is not stated; the plainest
# reading is used: score_j = Σ_i softmax_i(s)_j, the total attention
# probability each key receives over the reference queries.
# ---------------------------------------------------------------------------

def highest_attention_select(Q, K, t: int, scale=None, key_bias=None) -> List[int]:
    s = logits(Q, K, scale, key_bias)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    score = p.sum(axis=0)
    T = score.size
    order = np.lexsort((np.arange(T), -score))
    return [int(j) for j in order[:t]]


# ---------------------------------------------------------------------------
# Non-uniform head budgets by greedy swaps ([Summary] "Engineering
# Practicality": sensitivity curves rank head importance once, a greedy-swap
# algorithm assigns per-head ratios; [DeepDive] §4.2 steps 1-2; [News]
# "non-uniform compaction").  The pages name the algorithm only; the reading
# taken: one quantum at a time moves from the head that loses least by
# giving it up to the head that gains most by receiving it, while that
# lowers the summed loss, starting from the most even split.
# ---------------------------------------------------------------------------

def greedy_swap_budgets(loss, t_min: int, quantum: int, total: int,
                        max_swaps: Optional[int] = None):
    """Per-head budgets from sensitivity curves.

    loss[h][g] is head h's loss at budget t_min + g·quantum.  The levels
    start as even as the total allows (every head at units // H, one more
    for the first units % H heads, units = (total − H·t_min) / quantum).
    Each swap: the receiver b is the head with the largest gain
    loss[b][l_b] − loss[b][l_b + 1] (lowest index on ties, a head already at
    the top level excluded); the donor a is the head other than b with the
    smallest cost loss[a][l_a − 1] − loss[a][l_a] (lowest index on ties, a
    head at level 0 excluded); the quantum moves when gain > cost.  Returns
    (budgets, swaps)."""
    L = np.asarray(loss, F64)
    H, G = L.shape
    rest = total - H * t_min
    if rest < 0 or rest % quantum or rest // quantum > H * (G - 1):
        raise ValueError("total is not reachable on this budget grid")
    units = rest // quantum
    lev = [units // H + (1 if h < units % H else 0) for h in range(H)]
    swaps = 0
    while max_swaps is None or swaps < max_swaps:
        b, gain = -1, -math.inf
        for h in range(H):
            if lev[h] < G - 1:
                gh = L[h, lev[h]] - L[h, lev[h] + 1]
                if gh > gain:
                    b, gain = h, gh
        a, cost = -1, math.inf
        for h in range(H):
            if h != b and lev[h] > 0:
                ch = L[h, lev[h] - 1] - L[h, lev[h]]
                if ch < cost:
                    a, cost = h, ch
        if a < 0 or b < 0 or not gain > cost:
            break
        lev[a] -= 1
        lev[b] += 1
        swaps += 1
    return [t_min + quantum * x for x in lev], swaps
