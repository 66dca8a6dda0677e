"""Pins of the oracle's tail merging (the permuted layout's last tiles): a
worked example done by hand, the rules the schedule must satisfy on random
inputs, and the special cases with a closed form (identical plans pack by rows
alone; disjoint plans of whole KV tiles never merge)."""
import numpy as np
import pytest

import oracle


def _merge(sizes, plans, k_block=64):
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    idx = np.asarray(plans, np.int32)[None, None]
    return oracle.tail_merge(off, idx, k_block)[0]


def test_worked_example():
    # clusters of 50, 50, 200 and 30 rows: tails 50, 50, 72, 30 rows (slots 64,
    # 64, 96, 32), taken as g2, g0, g1, g3.  With 2 blocks per KV tile:
    #   g2 {7,8,9,10} opens tile 0 (96 rows);
    #   g0 {1,2,3,4}: no room in tile 0 (96 + 64 > 128) -> opens tile 1;
    #   g1 {1,2,3,5}: tile 1: union {1..5} needs 3 < 2 + 2 KV tiles -> joins at
    #      row 64;
    #   g3 {1,2,9,10}: tile 0 (96 + 32 rows fit): union {1,2,7,8,9,10} needs
    #      3 < 4 -> joins at row 96; tile 1 is full.
    mem, slo, ul, un = _merge([50, 50, 200, 30], [[1, 2, 3, 4], [1, 2, 3, 5], [7, 8, 9, 10], [1, 2, 9, 10]])
    assert mem.tolist() == [[2, 3, -1, -1], [0, 1, -1, -1]]
    assert slo.tolist() == [[0, 96, -1, -1], [0, 64, -1, -1]]
    assert ul.tolist() == [6, 5]
    assert un[0, :6].tolist() == [1, 2, 7, 8, 9, 10]
    assert un[1, :5].tolist() == [1, 2, 3, 4, 5]


def test_no_room_no_merge():
    # the same plans with tails of 72 and 40 rows (slots 96 and 64) cannot share
    mem, slo, ul, un = _merge([200, 40], [[7, 8, 9, 10], [7, 8, 9, 11]])
    assert mem.tolist() == [[0, -1, -1, -1], [1, -1, -1, -1]]


def test_joins_the_hamming_nearest_tile():
    # g0 {1,2,3,4} and g1 {1,2,10,11} (90-row tails, 96-row slots) open a
    # tile each, since both do not fit in one.  g2 {1,2,10,12} (a 20-row tail,
    # slot 32) fits in either, and either union saves a KV tile; it is at
    # Hamming distance 4 from tile 0 and 2 from tile 1, so it joins tile 1
    # although tile 0 was opened first.
    mem, slo, ul, un = _merge([90, 90, 20], [[1, 2, 3, 4], [1, 2, 10, 11], [1, 2, 10, 12]])
    assert mem.tolist() == [[0, -1, -1, -1], [1, 2, -1, -1]]
    assert slo.tolist() == [[0, -1, -1, -1], [0, 96, -1, -1]]
    assert un[1, :ul[1]].tolist() == [1, 2, 10, 11, 12]


def test_equal_distances_go_to_the_tile_opened_first():
    # as above, but g2 {1,2,7,8} is at Hamming distance 4 from both tiles
    mem, slo, ul, un = _merge([90, 90, 20], [[1, 2, 3, 4], [1, 2, 5, 6], [1, 2, 7, 8]])
    assert mem.tolist() == [[0, 2, -1, -1], [1, -1, -1, -1]]
    assert un[0, :ul[0]].tolist() == [1, 2, 3, 4, 7, 8]


def test_nearest_is_hamming_not_largest_overlap():
    # one block per KV tile (k_block 128): any overlap saves work.  Tails of
    # 30, 29, 28, 27 and 26 rows (one 32-row slot each), taken in that order:
    #   g0 {1,2,3,4} opens tile 0; g1 {30,31,32,33} shares nothing: tile 1;
    #   g2 {1,2,5,6} joins tile 0 (U = {1..6}); g3 {1,2,7,8} joins tile 0
    #   (U = {1..8}; tile 1 shares nothing);
    #   g4 {1,2,30,40} overlaps tile 0 in 2 blocks (distance 8 + 4 - 4 = 8) and
    #   tile 1 in 1 block (distance 4 + 4 - 2 = 6): it joins tile 1.
    mem, slo, ul, un = _merge([30, 29, 28, 27, 26],
                              [[1, 2, 3, 4], [30, 31, 32, 33], [1, 2, 5, 6], [1, 2, 7, 8], [1, 2, 30, 40]],
                              k_block=128)
    assert mem.tolist() == [[0, 2, 3, -1], [1, 4, -1, -1]]
    assert slo.tolist() == [[0, 32, 64, -1], [0, 32, -1, -1]]
    assert un[0, :ul[0]].tolist() == [1, 2, 3, 4, 5, 6, 7, 8]
    assert un[1, :ul[1]].tolist() == [1, 2, 30, 31, 32, 33, 40]


def test_identical_plans_pack_by_rows():
    # every union is the plan itself, so a tail joins the first tile with room
    # (all are at distance 0); 30-row tails take 32-row slots, four to a tile
    sizes = [30] * 10
    plans = [[5, 6, 7, 8]] * 10
    mem, slo, ul, un = _merge(sizes, plans)
    assert len(mem) == 3
    assert mem.tolist() == [[0, 1, 2, 3], [4, 5, 6, 7], [8, 9, -1, -1]]
    assert slo[0].tolist() == [0, 32, 64, 96]
    assert ul.tolist() == [4, 4, 4]


def test_disjoint_whole_tile_plans_never_merge():
    rng = np.random.default_rng(5)
    sizes = rng.integers(10, 300, 30)
    plans = np.arange(30 * 6).reshape(30, 6)  # 6 blocks = 3 whole KV tiles each, no overlap
    mem, slo, ul, un = _merge(sizes, plans)
    assert np.all(mem[:, 1] == -1)
    assert len(mem) == int(np.count_nonzero(sizes % 128))


@pytest.mark.parametrize("seed,k_block", [(0, 64), (1, 64), (2, 16), (3, 32), (4, 128)])
def test_schedule_rules_on_random_inputs(seed, k_block):
    rng = np.random.default_rng(seed)
    G, nK, S = 80, 200, 24
    sizes = np.clip(rng.zipf(1.3, G), 1, 700)
    pool = rng.permutation(nK)[:60]  # plans overlap: drawn from a shared pool plus their own blocks
    plans = []
    for g in range(G):
        own = rng.choice(nK, S, replace=False)
        shared = rng.choice(pool, S // 2, replace=False)
        p = list(dict.fromkeys(list(shared) + list(own)))[:S]
        plans.append(p)
    plans = np.array(plans, np.int32)
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    mem, slo, ul, un = oracle.tail_merge(off, plans[None, None], k_block)[0]
    b = 128 // k_block
    tails = {g: int(sizes[g] % 128) for g in range(G) if sizes[g] % 128}
    seen = []
    for t in range(len(mem)):
        ms = [int(m) for m in mem[t] if m >= 0]
        ss = [int(x) for x in slo[t][:len(ms)]]
        assert 1 <= len(ms) <= 4
        seen += ms
        # slots: whole 32-row quarters, in join order, back to back, inside the tile
        pos = 0
        for m, s0 in zip(ms, ss):
            assert s0 == pos and s0 % 32 == 0
            pos += (tails[m] + 31) // 32 * 32
        assert pos <= 128
        # the union is the members' plans, ascending
        u = sorted(set(np.concatenate([plans[m] for m in ms]).tolist()))
        assert un[t, :ul[t]].tolist() == u
        # merging never costs KV tiles: fewer than the members apart
        if len(ms) > 1:
            assert -(-len(u) // b) < sum(-(-len(set(plans[m].tolist())) // b) for m in ms)
    assert sorted(seen) == sorted(tails)
