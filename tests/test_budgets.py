"""Non-uniform head budgets by greedy swaps (host code, no GPU).

The oracle's greedy swap is pinned to the mathematics: on convex sensitivity
curves (diminishing returns) no single-quantum transfer can lower the summed
loss at its fixed point, which for a separable convex objective under a sum
constraint is the global minimum, checked here by enumerating every
assignment of small instances.  The library's C routine must then return the
oracle's budgets and swap count exactly (same rule, same float64 arithmetic).
"""
import itertools

import numpy as np
import pytest

import attention_matching_b200 as am
from attention_matching_b200 import workloads as W
from oracle import am_oracle as O


def convex_curves(rng, H, G):
    """Decreasing curves with shrinking decrements (convex), random scales."""
    out = np.empty((H, G))
    for h in range(H):
        dec = np.sort(rng.uniform(0.0, 1.0, G - 1))[::-1] * rng.uniform(0.1, 3.0)
        out[h] = rng.uniform(0.0, 1.0) + np.concatenate([[0.0], -np.cumsum(dec)]) + dec.sum()
    return out


def summed_loss(L, levels):
    return float(sum(L[h, g] for h, g in enumerate(levels)))


@pytest.mark.parametrize("seed", range(40))
def test_greedy_swap_reaches_the_enumerated_optimum_on_convex_curves(seed):
    rng = np.random.default_rng(seed)
    H, G = int(rng.integers(2, 5)), int(rng.integers(3, 7))
    L = convex_curves(rng, H, G)
    t_min, q = 4, 16
    for units in range(0, H * (G - 1) + 1):
        total = H * t_min + q * units
        budgets, _ = O.greedy_swap_budgets(L, t_min, q, total)
        lev = [(b - t_min) // q for b in budgets]
        best = min(summed_loss(L, c) for c in itertools.product(range(G), repeat=H) if sum(c) == units)
        assert summed_loss(L, lev) <= best + 1e-12, (seed, units, lev)


@pytest.mark.parametrize("convex", [True, False])
def test_greedy_swap_keeps_the_total_and_the_grid_and_lowers_the_loss(convex):
    L = W.sensitivity_curves(11, 16, 20, convex=convex)
    t_min, q = 4, 16
    total = 16 * t_min + q * 137
    budgets, swaps = O.greedy_swap_budgets(L, t_min, q, total)
    assert sum(budgets) == total and swaps >= 0
    lev = [(b - t_min) // q for b in budgets]
    assert all((b - t_min) % q == 0 and 0 <= x < 20 for b, x in zip(budgets, lev))
    even = [137 // 16 + (1 if h < 137 % 16 else 0) for h in range(16)]
    assert summed_loss(L, lev) <= summed_loss(L, even)
    # no improving transfer is left
    for a in range(16):
        for b in range(16):
            if a != b and lev[a] > 0 and lev[b] < 19:
                gain = L[b, lev[b]] - L[b, lev[b] + 1]
                cost = L[a, lev[a] - 1] - L[a, lev[a]]
                if convex:
                    assert not gain > cost + 1e-12


@pytest.mark.parametrize("H,G,units,convex,cap", [
    (1, 5, 3, True, None), (8, 64, 200, True, None), (64, 32, 900, False, None),
    (288, 64, 2949, True, None), (288, 64, 2949, False, None), (32, 16, 100, True, 7),
])
def test_library_matches_the_oracle_exactly(H, G, units, convex, cap):
    L = W.sensitivity_curves(100 + H + G, H, G, convex=convex)
    total = 4 * H + 16 * units
    want = O.greedy_swap_budgets(L, 4, 16, total, max_swaps=cap)
    got = am.assign_budgets(L, 4, 16, total, max_swaps=cap)
    assert got == (want[0], want[1])


def test_assign_budgets_argument_errors():
    L = W.sensitivity_curves(3, 4, 8)
    code = {v: k for k, v in am.STATUS.items()}
    with pytest.raises(am.AmError) as e:
        am.assign_budgets(L, 4, 16, 4 * 4 + 17)          # not on the grid
    assert e.value.code == code["AM_ERR_BUDGET"]
    with pytest.raises(am.AmError) as e:
        am.assign_budgets(L, 4, 16, 4 * 4 + 16 * 4 * 8)  # beyond the top level
    assert e.value.code == code["AM_ERR_BUDGET"]
    bad = L.copy()
    bad[1, 2] = np.nan
    with pytest.raises(am.AmError) as e:
        am.assign_budgets(bad, 4, 16, 4 * 4 + 16 * 5)
    assert e.value.code == code["AM_ERR_NONFINITE"]
