"""Pins of the oracle's selector (exact set + SIP sample) against what the pages
and probability theory fix: brute-force top-k, the capped-PPS inclusion
probabilities (sum, cap, proportionality, minimality), exact inclusion and
exact unbiasedness of the weighted numerator and denominator by integration
over the uniform, Monte-Carlo inclusion frequencies, and the pages' worked
example (probability one quarter counts four times)."""
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "sip_worked_example.txt")


def _row(rng, nK, kind="lognormal"):
    if kind == "lognormal":
        return np.exp(rng.normal(0, 1.5, nK)).astype(np.float32)
    if kind == "ties":
        return rng.integers(0, 4, nK).astype(np.float32)
    if kind == "spiky":
        m = rng.random(nK).astype(np.float32) * 0.01
        m[rng.choice(nK, 3, replace=False)] = 50.0
        return m
    raise ValueError(kind)


def _sample(m, ne, ns, U):
    idx, lw, pi, bad = oracle.select_row(m, ne, ns, U)
    return idx, lw, pi


@pytest.mark.parametrize("kind", ["lognormal", "ties", "spiky"])
def test_exact_set_is_bruteforce_topk(kind):
    rng = np.random.default_rng(5)
    for trial in range(50):
        nK = int(rng.integers(4, 40))
        m = _row(rng, nK, kind)
        ne = int(rng.integers(0, nK + 1))
        ns = int(rng.integers(0, nK - ne + 1))
        idx, lw, pi = _sample(m, ne, ns, int(rng.integers(0, 2**32)))
        brute = sorted(range(nK), key=lambda b: (-float(m[b]), b))[:ne]
        assert list(idx[:ne]) == sorted(brute)
        assert np.all(lw[:ne] == 0)


@pytest.mark.parametrize("kind", ["lognormal", "ties", "spiky"])
def test_plan_row_is_fixed_size_distinct_canonical(kind):
    rng = np.random.default_rng(6)
    for trial in range(50):
        nK = int(rng.integers(4, 60))
        m = _row(rng, nK, kind)
        ne = int(rng.integers(0, nK // 2 + 1))
        ns = int(rng.integers(0, nK - ne + 1))
        idx, lw, pi = _sample(m, ne, ns, int(rng.integers(0, 2**32)))
        assert len(idx) == ne + ns
        assert len(set(idx.tolist())) == ne + ns
        assert np.all((idx >= 0) & (idx < nK))
        assert np.all(np.diff(idx[:ne]) > 0) and np.all(np.diff(idx[ne:]) > 0)
        assert np.all(lw >= 0)


def _check_capped_pps(m, ne, ns, pi):
    """The capped PPS probabilities are the unique pi with: pi = 1 on the
    exact set, sum over the rest = n_s, pi <= 1, pi proportional to mass
    among the uncapped blocks, and every uncapped block strictly below 1
    (no block is capped that need not be)."""
    nK = len(m)
    brute = sorted(range(nK), key=lambda b: (-float(m[b]), b))[:ne]
    rest = [b for b in range(nK) if b not in set(brute)]
    assert np.all(pi[brute] == 1.0)
    if not rest:
        return
    assert abs(pi[rest].sum() - min(ns, len(rest))) < 1e-9 * max(1, ns)
    assert np.all(pi[rest] <= 1.0 + 1e-12)
    if ns == 0 or ns >= len(rest):
        return
    unc = [b for b in rest if pi[b] < 1.0]
    cap = [b for b in rest if pi[b] >= 1.0]
    mmax = max(float(m[b]) for b in rest)
    if mmax > 0 and unc:
        # pi = c * w with w in (x 2^31, x 2^31 + 1], x = m / m_max: the
        # quantised weights admit one common constant c for all uncapped blocks
        x = np.array([float(m[b]) / mmax for b in unc]) * 2.0**31
        p = np.array([pi[b] for b in unc])
        c_lo = p / (x + 1.0)
        c_hi = np.where(x > 0, p / np.maximum(x, 1e-300), np.inf)
        assert c_lo.max() <= c_hi.min() * (1 + 1e-12)
    if cap and unc:
        assert min(float(m[b]) for b in cap) >= max(float(m[b]) for b in unc)


@pytest.mark.parametrize("kind", ["lognormal", "ties", "spiky"])
def test_inclusion_probabilities_are_capped_pps(kind):
    rng = np.random.default_rng(7)
    for trial in range(60):
        nK = int(rng.integers(4, 60))
        m = _row(rng, nK, kind)
        ne = int(rng.integers(0, nK // 2 + 1))
        ns = int(rng.integers(0, nK - ne + 1))
        _, _, pi = _sample(m, ne, ns, 0)
        _check_capped_pps(m, ne, ns, pi)


def test_capping_engages_on_dominant_blocks():
    m = np.array([100.0, 90.0, 1.0, 1.0, 1.0, 1.0, 1.0, 1.0], np.float32)
    _, _, pi = _sample(m, 0, 3, 0)
    assert pi[0] == 1.0 and pi[1] == 1.0
    assert abs(pi[2:].sum() - 1.0) < 1e-12
    assert np.allclose(pi[2:], 1.0 / 6)


def _pieces(m, ne, ns):
    """The sample is a step function of U with breakpoints where a systematic
    point crosses a cumulative-weight boundary; each of the n' points moves
    monotonically with U, so the sample never recurs and bisection finds
    every breakpoint.  Returns [(U_start, U_end, idx, log_w)]."""
    key = lambda U: tuple(_sample(m, ne, ns, U)[0])
    out, U0 = [], 0
    while U0 < 2**32:
        s0 = key(U0)
        lo, hi = U0, 2**32  # sample(lo) == s0; hi is past the piece
        while hi - lo > 1:
            mid = (lo + hi) // 2
            if key(mid) == s0:
                lo = mid
            else:
                hi = mid
        idx, lw, _ = _sample(m, ne, ns, U0)
        out.append((U0, hi, idx, lw))
        U0 = hi
    return out


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_exact_inclusion_and_unbiased_numerator_denominator(seed):
    rng = np.random.default_rng(100 + seed)
    nK = int(rng.integers(10, 24))
    m = _row(rng, nK, "lognormal")
    ne = int(rng.integers(1, 4))
    ns = int(rng.integers(2, 6))
    _, _, pi = _sample(m, ne, ns, 0)
    pieces = _pieces(m, ne, ns)
    assert len(pieces) <= nK + 2
    incl = np.zeros(nK)
    # fixed "activations": per-block softmax denominators e_b > 0 and value sums a_b
    e = rng.random(nK) + 0.1
    a = rng.normal(size=(nK, 3))
    D_hat = 0.0
    N_hat = np.zeros(3)
    for U0, U1, idx, lw in pieces:
        p = (U1 - U0) / 2.0**32
        incl[idx] += p
        w = np.exp(lw.astype(np.float64))   # logit shift ln(1/pi) == weight 1/pi
        D_hat += p * np.sum(w * e[idx])
        N_hat += p * np.sum(w[:, None] * a[idx], axis=0)
    tol = (len(pieces) + 1) * 2.0**-32
    assert np.max(np.abs(incl - pi)) < tol + 1e-12
    # Horvitz-Thompson: numerator and denominator are individually unbiased
    assert abs(D_hat - e.sum()) < 1e-6 * e.sum()
    assert np.allclose(N_hat, a.sum(axis=0), atol=1e-6 * np.abs(a).sum())


def test_ratio_estimate_is_not_claimed_unbiased():
    """The pages state the normalised output is generally biased; the
    expectation of the ratio differs from the dense ratio on a skewed row."""
    m = np.array([8.0, 1.0, 1.0, 1.0, 1.0, 0.5], np.float32)
    pieces = _pieces(m, 0, 2)
    e = np.array([8.0, 3.0, 0.2, 1.0, 0.5, 4.0])     # true activations differ from the estimate
    a = np.array([1.0, -1.0, 0.0, 2.0, 0.0, 5.0])
    ratio = 0.0
    for U0, U1, idx, lw in pieces:
        w = np.exp(lw.astype(np.float64))
        ratio += (U1 - U0) / 2.0**32 * np.sum(w * e[idx] * a[idx]) / np.sum(w * e[idx])
    dense = np.sum(e * a) / np.sum(e)
    assert abs(ratio - dense) > 1e-3


def test_monte_carlo_inclusion_frequencies():
    rng = np.random.default_rng(3)
    nK = 16
    m = _row(rng, nK, "lognormal")
    ne, ns = 2, 4
    M = 20000
    mass = np.tile(m, (M, 1)).reshape(1, 1, M, nK)  # one row per group -> its own Philox draw
    idx, lw, bad = oracle.select(mass, ne, ns, seed=99)
    freq = np.zeros(nK)
    for row in idx.reshape(M, -1):
        freq[row] += 1
    freq /= M
    _, _, pi = _sample(m, ne, ns, 0)
    assert np.all(np.abs(freq - pi) <= 5 * np.sqrt(pi * (1 - pi) / M) + 1.0 / M)


def test_worked_example_quarter_counts_four_times():
    with open(GOLDEN) as f:
        p, mult = [float(x) for x in next(l for l in f if not l.startswith("#")).split()]
    # four equal blocks, one sampled: each enters with probability 1/4
    m = np.ones(4, np.float32)
    for U in [0, 2**30, 2**31, 3 * 2**30, 2**32 - 1]:
        idx, lw, pi = _sample(m, 0, 1, U)
        assert np.allclose(pi, p)
        assert math.isclose(math.exp(float(lw[0])), mult, rel_tol=1e-6)
    # and inside a larger row: an exact block plus a quarter-probability block
    m = np.array([10.0, 1.0, 1.0, 1.0, 1.0, 0.0], np.float32)
    idx, lw, pi = _sample(m, 1, 1, 123456789)
    assert idx[0] == 0 and np.allclose(pi[1:5], 0.25, atol=1e-9)
    assert math.isclose(math.exp(float(lw[1])), 4.0, rel_tol=1e-6)


def test_edge_cases():
    m = np.array([3.0, 1.0, 2.0, 0.0], np.float32)
    idx, lw, pi = _sample(m, 2, 0, 7)           # exact only
    assert list(idx) == [0, 2] and np.all(lw == 0)
    idx, lw, pi = _sample(m, 1, 3, 7)           # everything: dense plan, no weights
    assert list(idx) == [0, 1, 2, 3] and np.all(lw == 0)
    idx, lw, pi = _sample(np.zeros(8, np.float32), 2, 3, 5)   # all-zero mass: uniform PPS
    assert list(idx[:2]) == [0, 1]
    assert np.allclose(pi[2:], 3 / 6)
    mm = np.array([1.0, np.nan, 2.0, np.inf, 0.5, 0.25], np.float32)
    idx, lw, pi, bad = oracle.select_row(mm, 1, 2, 3)
    assert bad and idx[0] == 2
    with pytest.raises(ValueError):
        oracle.select_row(m, 3, 2, 0)


def test_non_positive_mass_counts_as_zero():
    # a mass estimate carries no weight below zero: negative entries select exactly
    # like zeros, for every split and uniform
    rng = np.random.default_rng(12)
    for _ in range(20):
        m = rng.normal(0.0, 1.0, 40).astype(np.float32)
        z = np.where(m > 0, m, 0.0).astype(np.float32)
        for ne, ns in [(5, 10), (0, 12), (20, 20)]:
            U = int(rng.integers(0, 2 ** 32))
            a = oracle.select_row(m, ne, ns, U)
            b = oracle.select_row(z, ne, ns, U)
            assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1]) and not a[3]
