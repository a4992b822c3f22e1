"""The rule behind the default correlation pass, checked on the host.

Split the queries into groups g (the residual update's: queries i with
(i / 128) mod G == g).  For every key, by Cauchy-Schwarz on each group,
|c_j| = |Σ_i r_i Φ_ij| <= Σ_g ‖r_g‖·‖Φ_{g,j}‖ = b_j.  A pass takes b_j for every
unselected key (group norms from fp32 partial sums of 32 squares raised by
1 + 2e-6 and stored in fp32, ‖r_g‖ from the fp64 residual, b_j stored fp32),
evaluates exactly the keys with b_j >= τ (τ: the lower edge of the
fp32-exponent histogram bin at which 2·kk + 32 keys are reached from the top),
takes θ = the kk-th largest value; when θ >= τ(1 + 1e-6) those are the picks,
otherwise it also evaluates the keys with b_j < τ and b_j(1 + 1e-6) >= θ and
takes the kk largest of everything evaluated.  The correlations themselves
are fp64 sums of the fp32 features times the fp32 copy of the residual.  These
tests restate that procedure and check that it always picks what a full pass
over every key picks (ties to the lower key), including residuals nearly
parallel to a feature column on one group, where the bound is tight.
"""
import numpy as np
import pytest

MARGIN = 1.0 + 1e-6
INFLATE = 1.0 + 2e-6


def group_norms(Phi32, G):
    """Per-group norm bounds as the library forms them: fp32 partial sums of
    32 squares, fp64 over the partials of a group, raised by 1 + 2e-6, fp32."""
    n, T = Phi32.shape
    sq = Phi32.astype(np.float32) ** 2
    pad = (-n) % 32
    sqp = np.concatenate([sq, np.zeros((pad, T), np.float32)]) if pad else sq
    part = sqp.reshape(-1, 32, T).sum(axis=1, dtype=np.float32).astype(np.float64)
    part_g = (np.arange(part.shape[0]) * 32 // 128) % G
    gn = np.stack([np.sqrt(part[part_g == g].sum(axis=0)) for g in range(G)])
    return (gn * INFLATE).astype(np.float32)


def bounds(gn32, r64, G):
    n = r64.size
    g_of = (np.arange(n) // 128) % G
    rg = np.sqrt(np.array([(r64[g_of == g] ** 2).sum() for g in range(G)]))
    return (rg[:, None] * gn32.astype(np.float64)).sum(axis=0).astype(np.float32)


def tau_for(b, target):
    pos = b[b > 0]
    if pos.size < target:
        return np.float32(0.0)
    bins = pos.view(np.uint32) >> 21
    hist = np.bincount(bins, minlength=1024)
    cum = np.cumsum(hist[::-1])
    k = int(np.argmax(cum >= target))
    return np.array([(1023 - k) << 21], dtype=np.uint32).view(np.float32)[0]


def top_kk(c, keys, kk):
    keys = np.asarray(sorted(keys))
    order = np.lexsort((keys, -c[keys]))
    return [int(keys[i]) for i in order[:kk]]


def bounded_pass(Phi32, r64, selected, kk, G):
    """(picks, number of rows evaluated)."""
    T = Phi32.shape[1]
    c = Phi32.astype(np.float64).T @ r64.astype(np.float32).astype(np.float64)
    b = bounds(group_norms(Phi32, G), r64, G)
    b[selected] = -1.0
    free = ~selected
    tau = tau_for(b, 2 * kk + 32)
    probe = np.flatnonzero(free & (b >= tau))
    top = top_kk(c, probe, kk)
    theta = c[top[kk - 1]] if len(top) >= kk else -np.inf
    if not tau > 0 or (len(top) >= kk and theta >= float(tau) * MARGIN):
        return top, probe.size
    rest = np.flatnonzero(free & (b < tau) & (b.astype(np.float64) * MARGIN >= theta))
    return top_kk(c, np.concatenate([probe, rest]), kk), probe.size + rest.size


def full_pass(Phi32, r64, selected, kk):
    c = Phi32.astype(np.float64).T @ r64.astype(np.float32).astype(np.float64)
    return top_kk(c, np.flatnonzero(~selected), kk)


@pytest.mark.parametrize("seed", range(30))
def test_bounded_pass_picks_what_a_full_pass_picks(seed):
    rng = np.random.default_rng(seed)
    n, T = int(rng.integers(130, 1200)), int(rng.integers(200, 1500))
    G = min((n + 127) // 128, 64)
    # features concentrated on a few queries per key, as attention mass is
    Phi32 = (np.exp(rng.standard_normal((n, T)) * 1.5 - 4.0) * rng.uniform(0.2, 3.0, T)).astype(np.float32)
    sel = rng.random(T) < 0.05
    w = np.abs(rng.standard_normal(T)) * sel
    r64 = Phi32.astype(np.float64).sum(axis=1) - Phi32.astype(np.float64) @ w
    for kk in (1, 4, 8, 16):
        got, evaluated = bounded_pass(Phi32, r64, sel, kk, G)
        assert got == full_pass(Phi32, r64, sel, kk)
        assert evaluated <= T


@pytest.mark.parametrize("seed", range(20))
def test_tight_group_bound_cases(seed):
    """The residual sits in one query group and is almost a multiple of one
    feature column there: that key's correlation nearly equals its bound."""
    rng = np.random.default_rng(100 + seed)
    n, T, G = 512, 800, 4
    Phi32 = np.exp(rng.standard_normal((n, T)) * 0.5).astype(np.float32)
    j0 = int(rng.integers(0, T))
    g0 = int(rng.integers(0, G))
    r64 = np.zeros(n)
    rows = slice(128 * g0, 128 * g0 + 128)
    r64[rows] = Phi32[rows, j0].astype(np.float64) * rng.uniform(0.5, 2.0) + rng.standard_normal(128) * 1e-9
    sel = np.zeros(T, bool)
    for kk in (1, 4, 8):
        assert bounded_pass(Phi32, r64, sel, kk, G)[0] == full_pass(Phi32, r64, sel, kk)


def test_group_bound_holds_and_is_tight():
    rng = np.random.default_rng(7)
    n, T, G = 512, 50, 4
    Phi32 = np.exp(rng.standard_normal((n, T))).astype(np.float32)
    r64 = np.zeros(n)
    r64[128:256] = Phi32[128:256, 3].astype(np.float64) * 0.7
    c = Phi32.astype(np.float64).T @ r64.astype(np.float32).astype(np.float64)
    b = bounds(group_norms(Phi32, G), r64, G).astype(np.float64) * MARGIN
    assert np.all(np.abs(c) <= b)
    assert c[3] <= b[3] <= c[3] * (1 + 1e-5)


def test_fewer_keys_than_the_probe_target_evaluates_them_all():
    rng = np.random.default_rng(3)
    Phi32 = np.exp(rng.standard_normal((200, 40))).astype(np.float32)
    r64 = Phi32.astype(np.float64).sum(axis=1)
    sel = np.zeros(40, bool)
    got, evaluated = bounded_pass(Phi32, r64, sel, 4, 2)
    assert evaluated == 40 and got == full_pass(Phi32, r64, sel, 4)
