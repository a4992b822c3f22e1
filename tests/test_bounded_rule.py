"""The bound behind the default correlation pass, checked on the host.

For every key |c_j| = |Σ_i r_i Φ_ij| <= ‖r‖·‖Φ_{:,j}‖ (Cauchy-Schwarz).  The
pass sorts keys by their column norms rounded to fp32, computes exact values
for a probe prefix, takes θ = the kk-th largest, and evaluates only the keys
whose fp32 norm reaches fl32(θ / (‖r‖(1 + 1e-7))), with ‖r‖ taken from the
fp64 residual while the correlated residual is its fp32 copy.  These tests
check the consequence the picks rely on: every key beyond that prefix has
c_j < θ, so the kk largest values all lie inside it.  The cases include
residuals nearly parallel to a feature column, where Cauchy-Schwarz is tight.
"""
import numpy as np
import pytest

MARGIN = 1e-7


def prefix_rule(Phi32, r64, probe, kk):
    """(θ, L, sorted order, c) as the pass forms them, in float64 sums."""
    r32 = r64.astype(np.float32)
    c = Phi32.astype(np.float64).T @ r32.astype(np.float64)
    norms = np.sqrt((Phi32.astype(np.float64) ** 2).sum(axis=0))
    knorm = norms.astype(np.float32)                      # rounded to nearest
    order = np.lexsort((np.arange(knorm.size), -knorm))   # descending, ties to the lower key
    theta = np.sort(c[order[:probe]])[::-1][kk - 1]
    rn = np.sqrt((r64 ** 2).sum())
    thr = np.float32(theta / (rn * (1.0 + MARGIN)))
    L = int((knorm >= thr).sum()) if theta > 0 else knorm.size
    return theta, L, order, c


def check(Phi32, r64, probe, kk):
    theta, L, order, c = prefix_rule(Phi32, r64, probe, kk)
    beyond = order[L:]
    assert np.all(c[beyond] < theta), (theta, c[beyond].max())
    top = np.argsort(-c, kind="stable")[:kk]
    assert set(top) <= set(order[:L].tolist()) or theta <= 0


@pytest.mark.parametrize("seed", range(30))
def test_keys_beyond_the_prefix_cannot_reach_the_threshold(seed):
    rng = np.random.default_rng(seed)
    n, T = int(rng.integers(64, 400)), int(rng.integers(300, 1500))
    scale = rng.uniform(0.2, 3.0, T)
    Phi = np.exp(rng.standard_normal((n, T)) * 0.7 - 2.0) * scale
    Phi32 = Phi.astype(np.float32)
    w = np.abs(rng.standard_normal(T)) * (rng.random(T) < 0.05)
    r64 = Phi32.astype(np.float64).sum(axis=1) - Phi32.astype(np.float64) @ w   # a residual m − Φ_S w
    check(Phi32, r64, probe=min(T, 128), kk=int(rng.integers(1, 17)))


@pytest.mark.parametrize("seed", range(20))
def test_tight_cauchy_schwarz_cases(seed):
    """The residual is almost a multiple of one feature column, so that
    column's correlation nearly equals its bound; the margin must still keep
    every excluded key strictly below θ."""
    rng = np.random.default_rng(100 + seed)
    n, T = 256, 800
    Phi32 = np.exp(rng.standard_normal((n, T)) * 0.5).astype(np.float32)
    j0 = int(rng.integers(0, T))
    r64 = Phi32[:, j0].astype(np.float64) * rng.uniform(0.5, 2.0) + rng.standard_normal(n) * 1e-9
    for kk in (1, 4, 8):
        for probe in (kk, 64, 256):
            check(Phi32, r64, probe, kk)


# ---------------------------------------------------------------------------
# The group bound of the second launch: |c_j| <= Σ_g ‖r_g‖·‖Φ_{g,j}‖, with the
# queries split into groups g = (i / 128) mod G (the residual update's
# partial sums), group norms from fp32 partial sums of 32 squares raised by
# 1 + 2e-6 and stored in fp32, and the sum raised by 1 + 1e-6.  A key whose
# bound is below θ is skipped: its c_j must be below θ too.
# ---------------------------------------------------------------------------

def group_bound(Phi32, r64, G):
    n, T = Phi32.shape
    seg = np.arange(n) // 128
    g_of = seg % G
    # fp32 partial sums of 32 squares (one warp's rows), then fp64 over partials
    sq = (Phi32.astype(np.float32) ** 2)
    pad = (-n) % 32
    sqp = np.concatenate([sq, np.zeros((pad, T), np.float32)]) if pad else sq
    part = sqp.reshape(-1, 32, T).sum(axis=1, dtype=np.float32).astype(np.float64)   # [n/32, T]
    part_g = (np.arange(part.shape[0]) * 32 // 128) % G
    gn = np.zeros((G, T))
    for g in range(G):
        gn[g] = np.sqrt(part[part_g == g].sum(axis=0))
    gn32 = (gn * (1.0 + 2e-6)).astype(np.float32).astype(np.float64)
    rg = np.sqrt(np.array([(r64[g_of == g] ** 2).sum() for g in range(G)]))
    return (rg[:, None] * gn32).sum(axis=0) * (1.0 + 1e-6)


@pytest.mark.parametrize("seed", range(20))
def test_group_bound_never_excludes_a_key_that_reaches_theta(seed):
    rng = np.random.default_rng(300 + seed)
    n, T = int(rng.integers(130, 1200)), int(rng.integers(200, 900))
    G = min((n + 127) // 128, 64)
    # features concentrated on a few queries per key, as attention mass is
    Phi = np.exp(rng.standard_normal((n, T)) * 1.5 - 4.0)
    Phi32 = Phi.astype(np.float32)
    w = np.abs(rng.standard_normal(T)) * (rng.random(T) < 0.05)
    r64 = Phi32.astype(np.float64).sum(axis=1) - Phi32.astype(np.float64) @ w
    c = Phi32.astype(np.float64).T @ r64.astype(np.float32).astype(np.float64)
    bound = group_bound(Phi32, r64, G)
    assert np.all(np.abs(c) <= bound), np.max(np.abs(c) / bound)
    # tighter than the global bound, and usually much tighter
    glob = np.sqrt((r64 ** 2).sum()) * np.sqrt((Phi32.astype(np.float64) ** 2).sum(axis=0))
    assert np.all(bound <= glob * (1 + 1e-5))
    for kk in (1, 4, 16):
        theta = np.sort(c)[::-1][kk - 1]
        skipped = bound < theta
        assert np.all(c[skipped] < theta)


def test_group_bound_is_tight_when_the_residual_sits_in_one_group():
    """r supported on one group and parallel to one key's features there:
    that key's bound equals its correlation to within the margins."""
    rng = np.random.default_rng(7)
    n, T, G = 512, 50, 4
    Phi32 = np.exp(rng.standard_normal((n, T))).astype(np.float32)
    r64 = np.zeros(n)
    r64[128:256] = Phi32[128:256, 3].astype(np.float64) * 0.7
    c = Phi32.astype(np.float64).T @ r64.astype(np.float32).astype(np.float64)
    bound = group_bound(Phi32, r64, G)
    assert c[3] <= bound[3] <= c[3] * (1 + 1e-5)
