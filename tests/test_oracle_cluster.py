"""Pins of the oracle's token clustering (the permuted layout of permuted
block-sparse attention: "InstaGen", abstract; the SVG2 semantic-aware
permutation it is parameterised by):

  * one assignment round equals a brute-force nearest-centroid search in
    numpy, with exact ties going to the lower centroid;
  * the sort equals numpy's stable argsort of the labels, and the offsets
    equal the cumulative label counts;
  * the update equals numpy's per-cluster means; an empty cluster keeps its
    centroid;
  * one cluster gives the mean of all rows and the identity permutation;
  * the k-means objective never increases from one round to the next;
  * after enough rounds the result is a Lloyd fixed point (every label is
    its row's nearest centroid, every centroid its cluster's mean);
  * well-separated generated clusters whose initial rows fall in distinct
    clusters are recovered exactly;
  * a hand-worked one-round case fixes the initial rows (the reading's
    floor(c N / C)) and the tie rule.
"""
import numpy as np
import pytest

import oracle


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even float32 -> bf16 bit patterns."""
    u = np.ascontiguousarray(a, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _x(rng, n, d, scale=1.0):
    return bf16_bits(rng.normal(0.0, scale, (n, d)))


def test_assign_matches_brute_force():
    rng = np.random.default_rng(1)
    for n, d, C in [(40, 8, 5), (200, 16, 12), (64, 4, 64)]:
        xb = _x(rng, n, d)
        x = bf16_to_f64(xb)
        mu = rng.normal(0.0, 1.0, (C, d))
        lab, _ = oracle.cluster_assign(xb, mu)
        dist = ((x[:, None, :] - mu[None, :, :]) ** 2).sum(-1)
        assert np.array_equal(lab, np.argmin(dist, axis=1))  # argmin takes the first minimum


def test_assign_exact_ties_go_to_the_lower_centroid():
    rng = np.random.default_rng(2)
    xb = _x(rng, 30, 6)
    mu = rng.normal(0.0, 1.0, (4, 6))
    mu = np.concatenate([mu[:2], mu[1:2], mu[2:]])  # centroid 2 duplicates centroid 1
    lab, amb = oracle.cluster_assign(xb, mu)
    assert not np.any(lab == 2)
    assert np.all(amb[lab == 1])  # a zero margin is flagged


def test_sort_is_a_stable_counting_sort():
    rng = np.random.default_rng(3)
    for n, C in [(1, 1), (100, 7), (1000, 50)]:
        lab = rng.integers(0, C, n).astype(np.int32)
        perm, off = oracle.cluster_sort(lab, C)
        assert np.array_equal(perm, np.argsort(lab, kind="stable"))
        assert np.array_equal(off, np.concatenate([[0], np.cumsum(np.bincount(lab, minlength=C))]))


def test_update_is_the_cluster_mean():
    rng = np.random.default_rng(4)
    n, d, C = 300, 12, 9
    xb = _x(rng, n, d)
    x = bf16_to_f64(xb)
    lab = rng.integers(0, C - 1, n).astype(np.int32)  # cluster C - 1 stays empty
    mu0 = rng.normal(size=(C, d))
    mu, cnt = oracle.cluster_update(xb, lab, mu0)
    assert np.array_equal(cnt, np.bincount(lab, minlength=C))
    for c in range(C - 1):
        np.testing.assert_allclose(mu[c], x[lab == c].mean(0), rtol=1e-13, atol=1e-13)
    assert np.array_equal(mu[C - 1], mu0[C - 1])


def test_one_cluster():
    rng = np.random.default_rng(5)
    xb = _x(rng, 77, 8)[None, None]
    lab, perm, off, mu, _ = oracle.cluster_tokens(xb, 1, 2)
    assert np.all(lab == 0)
    assert np.array_equal(perm[0, 0], np.arange(77))
    assert list(off[0, 0]) == [0, 77]
    np.testing.assert_allclose(mu[0, 0, 0], bf16_to_f64(xb[0, 0]).mean(0), rtol=1e-13, atol=1e-13)


def _objective(x, lab, mu):
    return float(((x - mu[lab]) ** 2).sum())


def test_objective_never_increases():
    rng = np.random.default_rng(6)
    xb = _x(rng, 400, 8)
    x = bf16_to_f64(xb)
    J = []
    for it in range(1, 8):
        lab, _, _, mu, _ = oracle.cluster_tokens(xb[None, None], 10, it)
        J.append(_objective(x, lab[0, 0], mu[0, 0]))
    assert all(b <= a * (1 + 1e-12) for a, b in zip(J, J[1:])), J


def test_fixed_point_after_convergence():
    rng = np.random.default_rng(7)
    xb = _x(rng, 300, 6)
    x = bf16_to_f64(xb)
    lab, perm, off, mu, _ = oracle.cluster_tokens(xb[None, None], 6, 60)
    lab, perm, off, mu = lab[0, 0], perm[0, 0], off[0, 0], mu[0, 0]
    dist = ((x[:, None, :] - mu[None]) ** 2).sum(-1)
    assert np.array_equal(lab, np.argmin(dist, axis=1))
    for c in range(6):
        if np.any(lab == c):
            np.testing.assert_allclose(mu[c], x[lab == c].mean(0), rtol=1e-12, atol=1e-12)
    # the layout: labels sorted along the permutation, rows ascending within a cluster
    assert sorted(perm.tolist()) == list(range(300))
    assert np.all(np.diff(lab[perm]) >= 0)
    for c in range(6):
        seg = perm[off[c]:off[c + 1]]
        assert np.all(np.diff(seg) > 0) and np.all(lab[seg] == c)


def test_well_separated_clusters_are_recovered():
    rng = np.random.default_rng(8)
    C, per, d = 5, 40, 16
    centres = rng.normal(0.0, 10.0, (C, d))
    truth = np.repeat(np.arange(C), per)           # row floor(c N / C) is in cluster c
    x = centres[truth] + rng.normal(0.0, 0.1, (C * per, d))
    shuffle_inside = np.concatenate([rng.permutation(per) + c * per for c in range(C)])
    x = x[shuffle_inside]
    lab, perm, off, _, amb = oracle.cluster_tokens(bf16_bits(x)[None, None], C, 3)
    assert not amb[0, 0]
    assert np.array_equal(lab[0, 0], truth)
    assert np.array_equal(off[0, 0], np.arange(C + 1) * per)


def test_initial_centroids_are_rows_c_n_over_c():
    # one round from the initial centroids: rows 0, 2 and 4 of six (floor(c 6 / 3)),
    # worked by hand; the values are such that every other ordered choice of three
    # initial rows gives other labels or other means after the round
    x = np.array([[2.0], [9.0], [14.0], [17.0], [23.0], [38.0]])
    lab, perm, off, mu, _ = oracle.cluster_tokens(bf16_bits(x)[None, None], 3, 1)
    # centroids 2, 14, 23: 9 is 5 from 14 and 7 from 2; 17 is 3 from 14 and 6 from 23
    assert list(lab[0, 0]) == [0, 1, 1, 1, 2, 2]
    np.testing.assert_allclose(mu[0, 0, :, 0], [2.0, 40.0 / 3.0, 30.5], rtol=1e-15)
    # a tie goes to the lower centroid: 16 is 2 from both 14 and 18
    x = np.array([[14.0], [16.0], [18.0]])
    lab, _, _, _, amb = oracle.cluster_tokens(bf16_bits(x)[None, None], 2, 1)  # rows 0 and 1 start
    assert list(lab[0, 0]) == [0, 1, 1]
    lab2, _ = oracle.cluster_assign(bf16_bits(np.array([[16.0]])), np.array([[14.0], [18.0]]))
    assert list(lab2) == [0]


def test_arguments():
    with pytest.raises(ValueError):
        oracle.cluster_tokens(np.zeros((1, 1, 4, 2), np.uint16), 5, 1)
    with pytest.raises(ValueError):
        oracle.cluster_tokens(np.zeros((1, 1, 4, 2), np.uint16), 2, 0)
    with pytest.raises(ValueError):
        oracle.cluster_sort(np.array([0, 3], np.int32), 3)
