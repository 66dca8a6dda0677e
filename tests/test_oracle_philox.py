"""Pins of the oracle's Philox4x64-10 against numpy's implementation of the
same published generator and against the generator's known-answer vectors."""
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "philox4x64_10_kat.txt")


def _numpy_at(counter, key):
    """numpy's Philox bumps the counter before generating: start it one below."""
    c = [int(x) for x in counter]
    i = 0
    while True:  # subtract one with borrow
        if c[i] > 0:
            c[i] -= 1
            break
        c[i] = (1 << 64) - 1
        i += 1
        if i == 4:
            break
    bg = np.random.Philox(counter=np.array(c, dtype=np.uint64), key=np.array(key, dtype=np.uint64))
    return bg.random_raw(4)


def test_known_answer_vectors():
    with open(GOLDEN) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    assert len(rows) == 2
    for r in rows:
        v = [int(x, 16) for x in r]
        out = oracle.philox4x64_10(v[0:4], v[4:6])
        assert [int(x) for x in out] == v[6:10]


def test_matches_numpy_random_counters():
    rng = np.random.default_rng(1234)
    for _ in range(200):
        ctr = [int(x) for x in rng.integers(0, 2**63, 4, dtype=np.int64)]
        key = [int(x) for x in rng.integers(0, 2**63, 2, dtype=np.int64)]
        ctr[rng.integers(0, 4)] = 0  # include zero words (borrow path)
        assert [int(x) for x in oracle.philox4x64_10(ctr, key)] == [int(x) for x in _numpy_at(ctr, key)]


def test_group_uniform_is_high_word_of_output0():
    for seed, b, h, g in [(0, 0, 0, 0), (0, 0, 3, 17), (7, 1, 39, 590), (2**40 + 5, 0, 23, 928)]:
        raw = _numpy_at([g, h, b, 0], [seed, 0])
        assert oracle.group_uniform(seed, b, h, g) == int(raw[0]) >> 32


def test_group_uniform_is_uniform():
    us = np.array([oracle.group_uniform(11, 0, 0, g) for g in range(20000)], np.float64) / 2**32
    # mean and variance of U[0,1) within 6 sigma; a Kolmogorov-Smirnov distance bound
    assert abs(us.mean() - 0.5) < 6 * np.sqrt(1 / 12 / len(us))
    assert abs(us.var() - 1 / 12) < 0.01
    srt = np.sort(us)
    ks = np.max(np.abs(srt - (np.arange(len(us)) + 0.5) / len(us)))
    assert ks < 1.63 / np.sqrt(len(us)) + 1e-3
