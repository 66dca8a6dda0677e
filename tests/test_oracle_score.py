"""Pins of the oracle's block scorer (key means, in-group k-means, estimated
mass): plain-definition checks with numpy, brute force on tiny inputs,
Lloyd's fixed-point and monotonicity properties, the mass sum invariant and
the one-cluster closed form."""
import numpy as np
import torch

import oracle
from block_sparse_importance_b200 import workloads as wl


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _val(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_key_means_match_numpy_including_tail():
    rng = np.random.default_rng(0)
    for N, Bk in [(64, 16), (100, 16), (130, 64), (7, 64)]:
        k = _bf16_bits(rng.normal(size=(N, 32)))
        kbar, L = oracle.key_means(k, Bk)
        nK = -(-N // Bk)
        assert kbar.shape == (nK, 32) and L.sum() == N
        for b in range(nK):
            rows = _val(k[b * Bk:min(N, (b + 1) * Bk)])
            assert L[b] == len(rows)
            assert np.allclose(kbar[b], rows.mean(axis=0), rtol=0, atol=1e-13)


def _nearest(x, mu):
    d = ((x[:, None, :] - mu[None, :, :]) ** 2).sum(-1)
    return d.argmin(axis=1)  # argmin picks the lowest index on ties


def test_kmeans_one_iteration_bruteforce():
    rng = np.random.default_rng(1)
    for n, C in [(64, 4), (128, 8), (20, 3), (5, 8)]:
        q = _bf16_bits(rng.normal(size=(n, 16)))
        x = _val(q)
        mu, cnt, amb = oracle.kmeans_group(q, C, 1)
        init = x[[(c * n) // C for c in range(C)]]
        a = _nearest(x, init)
        assert list(cnt) == [int((a == c).sum()) for c in range(C)]
        for c in range(C):
            want = x[a == c].mean(axis=0) if (a == c).any() else init[c]
            assert np.allclose(mu[c], want, atol=1e-12)


def test_kmeans_invariants_and_monotone_objective():
    rng = np.random.default_rng(2)
    centres = rng.normal(size=(6, 32)) * 3
    x = centres[rng.integers(0, 6, 128)] + rng.normal(size=(128, 32))
    q = _bf16_bits(x)
    xv = _val(q)
    prev = np.inf
    for iters in [1, 2, 3, 5, 10, 40]:
        mu, cnt, amb = oracle.kmeans_group(q, 8, iters)
        assert cnt.sum() == 128
        # objective of the returned centroids under nearest assignment
        a = _nearest(xv, mu)
        obj = ((xv - mu[a]) ** 2).sum()
        assert obj <= prev + 1e-9
        prev = obj
    # after convergence Lloyd's map is at a fixed point
    a = _nearest(xv, mu)
    assert list(cnt) == [int((a == c).sum()) for c in range(8)]
    for c in range(8):
        if cnt[c]:
            assert np.allclose(mu[c], xv[a == c].mean(axis=0), atol=1e-12)


def test_kmeans_special_cases():
    rng = np.random.default_rng(3)
    q = _bf16_bits(rng.normal(size=(50, 8)))
    x = _val(q)
    mu, cnt, _ = oracle.kmeans_group(q, 1, 3)      # one cluster: the group mean
    assert cnt[0] == 50 and np.allclose(mu[0], x.mean(axis=0), atol=1e-13)
    q = _bf16_bits(np.eye(6, 8) * 4.0)              # distinct rows, one cluster each
    mu, cnt, _ = oracle.kmeans_group(q, 6, 3)
    assert list(cnt) == [1] * 6 and np.allclose(mu, _val(q))


def test_kmeans_near_tie_is_flagged():
    mu, cnt, amb = oracle.kmeans_group(_bf16_bits(np.array([[-1.0, 0.0], [0.0, 0.0], [1.0, 0.0]])), 2, 1)
    # init: rows 0 and 1 ( floor(0*3/2)=0, floor(1*3/2)=1 ); row 2 is nearest to row 1 -> no tie
    assert not amb
    mu, cnt, amb = oracle.kmeans_group(_bf16_bits(np.array([[-1.0, 0.0], [0.0, 0.0], [1.0, 0.0], [0.5, 1.0]])), 2, 1)
    # init rows 0 and 2 = (-1,0) and (1,0): row 1 (0,0) is equidistant -> tie, goes to c=0
    assert amb and cnt[0] == 2 and cnt[1] == 2


def test_mass_sums_to_group_size_and_single_cluster_closed_form():
    rng = np.random.default_rng(4)
    d, N, Bk, scale = 16, 100, 16, 0.25
    k = _bf16_bits(rng.normal(size=(N, d)))
    kbar, L = oracle.key_means(k, Bk)
    q = _bf16_bits(rng.normal(size=(40, d)))
    for C in [1, 3, 8]:
        mu, cnt, _ = oracle.kmeans_group(q, C, 3)
        m = oracle.mass_group(mu, cnt, kbar, L, scale)
        assert abs(m.sum() - 40) < 1e-10
        assert np.all(m >= 0)
    # C = 1: mu is the group mean and m = n * softmax_b(scale mu.kbar_b + ln L_b)
    mu, cnt, _ = oracle.kmeans_group(q, 1, 3)
    x = _val(q).mean(axis=0)
    z = scale * kbar @ x
    p = L * np.exp(z - z.max())
    assert np.allclose(oracle.mass_group(mu, cnt, kbar, L, scale), 40 * p / p.sum(), rtol=1e-12)
    # empty clusters contribute nothing
    mu2 = np.vstack([mu, 100 * np.ones((1, d))])
    assert np.allclose(oracle.mass_group(mu2, np.array([40, 0]), kbar, L, scale),
                       oracle.mass_group(mu, cnt, kbar, L, scale), rtol=0, atol=1e-12)


def test_score_driver_matches_per_group_functions():
    w = wl.preset("tiny")
    inp = wl.make_inputs(w, "cpu", seq_len=1000)
    q, k = wl.bf16_bits(inp.q), wl.bf16_bits(inp.k)
    off = inp.offsets
    mass, cen, cnt, amb = oracle.score(q, k, off, w.k_block, w.n_clusters, w.n_iters, w.scale)
    kbar, L = oracle.key_means(k[0, 0], w.k_block)
    for g in [0, 3, len(off) - 2]:
        mu, c, a = oracle.kmeans_group(q[0, 0, off[g]:off[g + 1]], w.n_clusters, w.n_iters)
        assert np.array_equal(c, cnt[0, 0, g]) and np.allclose(mu, cen[0, 0, g], atol=0)
        assert np.allclose(oracle.mass_group(mu, c, kbar, L, w.scale), mass[0, 0, g], atol=0)
        assert abs(mass[0, 0, g].sum() - (off[g + 1] - off[g])) < 1e-9
