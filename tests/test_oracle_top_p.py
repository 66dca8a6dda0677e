"""Pins of the oracle's top-p rule (exact-set size from a share of the mass;
"iCATS", Method summary: sparsity set by the share p of attention mass kept).

  * brute force: the size equals a plain Python count over the blocks sorted
    by mass (descending, ties to the lower block), with the same quantised
    integer masses and the same fp64 target, on rows with ties and zeros;
  * it never decreases as p grows, p = 1 keeps every block of positive
    weight (capped at S), and a row of zeros keeps none;
  * the plan it makes equals the fixed-size selector's plan with
    n_exact = k_e and n_sample = S - k_e, row by row, uniform included.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle


def brute_k(m: np.ndarray, p: float, S: int) -> int:
    """The fewest blocks, by descending mass, whose quantised sum reaches the
    share p of the row's total, compared as exact rationals (fl(p * total)
    is the product the reading rounds once in fp64)."""
    vals = [float(x) if (math.isfinite(float(x)) and float(x) > 0.0) else 0.0 for x in m]
    mmax = max(vals)
    q = [math.floor(v / mmax * 2147483648.0) if (v > 0.0 and mmax > 0.0) else 0 for v in vals]
    share = Fraction(p * float(sum(q)))
    order = sorted(range(len(vals)), key=lambda b: (-vals[b], b))
    k, cum = 0, 0
    while Fraction(cum) < share and k < len(vals):
        cum += q[order[k]]
        k += 1
    return min(k, S)


def _rows(rng, n_rows, nK):
    rows = []
    for i in range(n_rows):
        kind = i % 4
        if kind == 0:
            m = np.exp(rng.normal(0.0, 2.0, nK))
        elif kind == 1:
            m = rng.integers(0, 4, nK).astype(np.float64)       # ties and zeros
        elif kind == 2:
            m = rng.random(nK) * 1e-3
            m[rng.choice(nK, min(nK, 3), replace=False)] = 50.0  # a few dominant blocks
        else:
            m = np.zeros(nK)
            m[rng.integers(0, nK)] = 1.0
        rows.append(m.astype(np.float32))
    return rows


@pytest.mark.parametrize("nK,S", [(7, 5), (40, 12), (300, 60)])
@pytest.mark.parametrize("p", [0.05, 0.3, 0.5, 0.8, 0.95, 1.0])
def test_top_p_count_matches_brute_force(nK, S, p):
    rng = np.random.default_rng(nK + int(p * 100))
    for m in _rows(rng, 24, nK):
        k, bad = oracle.top_p_count(m, p, S)
        assert not bad
        assert k == brute_k(m, p, S)


def test_top_p_count_at_a_fractional_share():
    # two equal blocks, q = 2^31 each; p = 1/2 + 2^-33 puts the share at
    # 2^31 + 1/2: one block falls short by half a unit, so both are needed
    m = np.array([1.0, 1.0], np.float32)
    p = 0.5 + 2.0 ** -33
    assert p * 2.0 ** 32 == 2.0 ** 31 + 0.5
    assert oracle.top_p_count(m, p, 2)[0] == 2 == brute_k(m, p, 2)
    assert oracle.top_p_count(m, 0.5, 2)[0] == 1 == brute_k(m, 0.5, 2)


def test_top_p_count_edges():
    rng = np.random.default_rng(5)
    for m in _rows(rng, 40, 64):
        ks = [oracle.top_p_count(m, p, 64)[0] for p in (0.1, 0.25, 0.5, 0.75, 0.9, 1.0)]
        assert ks == sorted(ks)
        positive = int(np.sum(np.floor(m.astype(np.float64) / m.max() * 2147483648.0) > 0)) if m.max() > 0 else 0
        assert oracle.top_p_count(m, 1.0, 64)[0] == positive
        assert oracle.top_p_count(m, 1.0, 3)[0] == min(3, positive)
    assert oracle.top_p_count(np.zeros(10, np.float32), 0.9, 5)[0] == 0
    with pytest.raises(ValueError):
        oracle.top_p_count(np.ones(4, np.float32), 0.0, 2)
    with pytest.raises(ValueError):
        oracle.top_p_count(np.ones(4, np.float32), 1.5, 2)


def test_top_p_plan_equals_fixed_split_per_row():
    rng = np.random.default_rng(11)
    B, H, G, nK, S, seed = 1, 2, 5, 50, 16, 3
    mass = np.exp(rng.normal(0.0, 1.5, (B, H, G, nK))).astype(np.float32)
    idx, lw, ke, bad = oracle.select_top_p(mass, 0.6, S, seed)
    assert not bad
    for h in range(H):
        for g in range(G):
            k = int(ke[0, h, g])
            assert k == oracle.top_p_count(mass[0, h, g], 0.6, S)[0]
            U = oracle.group_uniform(seed, 0, h, g)
            i2, l2, _, _ = oracle.select_row(mass[0, h, g], k, S - k, U)
            assert np.array_equal(idx[0, h, g], i2)
            assert np.array_equal(lw[0, h, g], l2)
            # the exact part is the head of the plan, with zero log-weights
            assert np.all(lw[0, h, g, :k] == 0.0)
