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
