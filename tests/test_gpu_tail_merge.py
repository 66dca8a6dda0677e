"""GPU parity of tail merging (the permuted layout): the schedule isa_tail_merge
builds equals the oracle's bit for bit (tiles, members, slots, unions), and
isa_attention_merged matches the fp64 oracle's per-row attention (each row
keeps its own cluster's plan), on clustered inputs with oracle plans, for every
key-block size."""
import numpy as np
import pytest
import torch

import oracle
from tests import cases
from tests.cases import Case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def isa():
    from block_sparse_importance_b200 import build, isa as m
    build.build()
    return m


def _up(x):
    return (x + 255) & ~255


def _read_schedule(sched, BH, N, G, S, nK):
    """The tiles of each (b, h) from the schedule buffer.  Its parts follow one
    another, each rounded up to 256 bytes: tiles [BH][G] of 16 int32 (members,
    rows, union length, union offset, table offset, 3 unused, clusters[4],
    slots[4]); counts [BH][2] (tiles, merged tiles); scratch (the tails'
    order [BH][G], the greedy's state [BH][3 G + 2 W + G W] and word prefixes
    [BH][8][W], W = ceil(nK / 32)); the union pool [BH][G S]; the rest."""
    W = (nK + 31) // 32
    buf = sched.cpu().numpy().view(np.int32)
    o_bins = 0
    o_counts = o_bins + _up(BH * G * 64)
    o_order = o_counts + _up(BH * 8)
    o_state = o_order + _up(BH * G * 4)
    o_prefix = o_state + _up(BH * (3 * G + 2 * W + G * W) * 4)
    o_unions = o_prefix + _up(BH * 8 * W * 4)
    bins = buf[o_bins // 4: o_bins // 4 + BH * G * 16].reshape(BH, G, 16)
    counts = buf[o_counts // 4: o_counts // 4 + 2 * BH].reshape(BH, 2)
    unions = buf[o_unions // 4: o_unions // 4 + BH * G * S].reshape(BH, G * S)
    out = []
    for bh in range(BH):
        tiles = []
        for k in range(counts[bh, 0]):
            b = bins[bh, k]
            n, ulen, uoff = int(b[0]), int(b[2]), int(b[3])
            mem = [int(x) for x in b[8:12]]
            slo = [int(x) for x in b[12:16]]
            u = unions[bh, uoff:uoff + ulen].tolist() if n > 1 else None
            tiles.append((mem, slo, ulen, u))
        assert counts[bh, 1] == sum(1 for t in tiles if t[0][1] >= 0)
        out.append(tiles)
    return out


def _case(N, Bk, ne, ns, seed):
    off = cases.random_offsets(N, 8, 300, seed=seed)
    return Case("wan13", 2, N, Bk, 128, ne, ns, offsets=off, seed=seed)


@pytest.mark.parametrize("N,Bk,ne,ns,seed", [
    (3000, 64, 4, 6, 1),
    (2600, 16, 8, 16, 2),
    (2000, 32, 5, 6, 3),
    (1800, 128, 2, 3, 4),
])
def test_schedule_and_attention_match_oracle(isa, N, Bk, ne, ns, seed):
    c = _case(N, Bk, ne, ns, seed)
    idx, lw = c.plan()
    S = idx.shape[-1]
    lay = c.layout()
    q, k, v = c.cuda()
    idx_d, lw_d = torch.from_numpy(idx).cuda(), torch.from_numpy(lw).cuda()
    sched = isa.tail_merge(idx_d, lw_d, lay)
    assert isa.context().sync_status() == isa.ISA_OK
    # the schedule, bit for bit
    got = _read_schedule(sched, c.H, N, c.G, S, c.nK)
    ref = oracle.tail_merge(c.offsets, idx, Bk)
    multi = 0
    for bh in range(c.H):
        mem, slo, ul, un = ref[bh]
        assert len(got[bh]) == len(mem)
        for t, (gm, gs, gl, gu) in enumerate(got[bh]):
            assert gm == mem[t].tolist()
            assert gs == slo[t].tolist()
            assert gl == ul[t]
            if gm[1] >= 0:
                multi += 1
                assert gu == un[t, :ul[t]].tolist()
    assert multi > 0, "the case merges no tails"
    # the attention: every row on its own cluster's plan
    out, lse = isa.attention_merged(q, k, v, idx_d, lw_d, lay, sched, want_lse=True)
    assert isa.context().sync_status() == isa.ISA_OK
    ref_out, ref_lse = c.oracle_attention()
    cases.check_attention(out, ref_out, lse, ref_lse)
    # and the tile-by-tile pass gives the same rows within rounding
    out2, lse2 = isa.attention(q, k, v, idx_d, lw_d, lay, want_lse=True)
    assert isa.context().sync_status() == isa.ISA_OK
    d = (out.float() - out2.float()).abs().max().item()
    assert d <= 2 * cases.ATTN_MAX_ABS
    assert (lse - lse2).abs().max().item() < 2e-2


def test_merged_with_logit_jumps(isa):
    """A member whose first blocks in the union come late, and log-weights far
    above the running max: rows start their max at their first block."""
    c = _case(2400, 64, 4, 6, 7)
    idx, lw = c.plan()
    lw = lw.copy()
    S = lw.shape[-1]
    for h in range(c.H):
        for g in range(c.G):
            lw[0, h, g, (g * 7 + h) % S] += [0.0, 40.0, -60.0][(g + h) % 3]
    q, k, v = c.cuda()
    idx_d, lw_d = torch.from_numpy(idx).cuda(), torch.from_numpy(lw).cuda()
    lay = c.layout()
    sched = isa.tail_merge(idx_d, lw_d, lay)
    out, lse = isa.attention_merged(q, k, v, idx_d, lw_d, lay, sched, want_lse=True)
    assert isa.context().sync_status() == isa.ISA_OK
    ref_out, ref_lse = c.oracle_attention(idx, lw)
    cases.check_attention(out, ref_out, lse, ref_lse)


def test_merge_host_checks(isa):
    c = Case("wan13", 1, 600, 64, 128, 2, 2)  # uniform groups: no q_offsets
    idx, lw = c.plan()
    with pytest.raises(isa.IsaError):
        isa.tail_merge(torch.from_numpy(idx).cuda(), torch.from_numpy(lw).cuda(), c.layout())


def test_schedule_with_state_in_global_memory(isa):
    """About 1000 clusters of 8..30 rows over 1250 key blocks: the greedy's masks
    (G x 40 words) no longer fit in shared memory and live in the workspace."""
    N, Bk = 20000, 16
    off = cases.random_offsets(N, 8, 30, seed=11)
    c = Case("wan13", 1, N, Bk, 128, 4, 8, offsets=off, seed=11)
    G, W = c.G, (c.nK + 31) // 32
    assert (3 * G + 2 * W + G * W) * 4 > 160 * 1024
    idx, lw = c.plan()
    q, k, v = c.cuda()
    idx_d, lw_d = torch.from_numpy(idx).cuda(), torch.from_numpy(lw).cuda()
    lay = c.layout()
    sched = isa.tail_merge(idx_d, lw_d, lay)
    assert isa.context().sync_status() == isa.ISA_OK
    got = _read_schedule(sched, c.H, N, G, idx.shape[-1], c.nK)
    mem, slo, ul, un = oracle.tail_merge(c.offsets, idx, Bk)[0]
    assert [t[0] for t in got[0]] == mem.tolist()
    assert [t[1] for t in got[0]] == slo.tolist()
    assert [t[2] for t in got[0]] == ul.tolist()
    out, lse = isa.attention_merged(q, k, v, idx_d, lw_d, lay, sched, want_lse=True)
    assert isa.context().sync_status() == isa.ISA_OK
    ref_out, ref_lse = c.oracle_attention()
    cases.check_attention(out, ref_out, lse, ref_lse)


def test_full_layer_varclust(isa):
    """The permuted layout at its full size (40 heads, 75 600 rows in 600
    clusters, as the benchmark's tail-merge run): the oracle's plans of the
    first and last head are placed in the layer's plan, isa_tail_merge runs on
    the whole layer, and for those heads the schedule equals the oracle's bit
    for bit and the merged attention of sampled clusters (members of merged
    tiles and clusters left alone) matches the oracle."""
    from block_sparse_importance_b200 import workloads as wl
    w = wl.preset("varclust")
    inp = wl.make_inputs(w, "cuda")
    q, k, v = inp.q, inp.k, inp.v
    B, H, N, d = q.shape
    off = inp.offsets
    lay = isa.layout_for(q, w.k_block, w.q_block, q_offsets=torch.from_numpy(off).cuda(), scale=w.scale)
    G, nK, S = lay.num_groups, lay.n_key_blocks, w.n_select
    mass = isa.score(q, k, lay, w.n_clusters, w.n_iters)
    idx, lw = isa.select(mass, lay, w.n_exact, w.n_sample, w.seed)
    assert isa.context().sync_status() == isa.ISA_OK

    heads = [0, H - 1]
    qb = wl.bf16_bits(q[:, heads])
    kb = wl.bf16_bits(k[:, heads])
    vb = wl.bf16_bits(v[:, heads])
    m_ref, _, _, _ = oracle.score(qb, kb, off, w.k_block, w.n_clusters, w.n_iters, w.scale)
    idx_ref, lw_ref, _ = oracle.select(m_ref.astype(np.float32), w.n_exact, w.n_sample, w.seed)
    for j, hh in enumerate(heads):
        idx[:, hh] = torch.from_numpy(idx_ref[:, j]).cuda()
        lw[:, hh] = torch.from_numpy(lw_ref[:, j]).cuda()

    sched = isa.tail_merge(idx, lw, lay)
    assert isa.context().sync_status() == isa.ISA_OK
    got = _read_schedule(sched, H, N, G, S, nK)
    ref = oracle.tail_merge(off, idx_ref, w.k_block)
    rng = np.random.default_rng(5)
    sample = []
    for j, hh in enumerate(heads):
        mem, slo, ul, un = ref[j]
        tiles = got[hh]
        assert len(tiles) == len(mem)
        n_multi = 0
        for t, (gm, gs, gl, gu) in enumerate(tiles):
            assert gm == mem[t].tolist()
            assert gs == slo[t].tolist()
            assert gl == ul[t]
            if gm[1] >= 0:
                n_multi += 1
                assert gu == un[t, :ul[t]].tolist()
        assert n_multi > 50
        merged = sorted({g for gm, _, _, _ in tiles if gm[1] >= 0 for g in gm if g >= 0})
        alone = sorted(set(range(G)) - set(merged))
        pick = list(rng.choice(merged, 24, replace=False)) + list(rng.choice(alone, 8, replace=False))
        sample += [(0, j, int(g)) for g in sorted(pick)]

    out, lse = isa.attention_merged(q, k, v, idx, lw, lay, sched, want_lse=True)
    assert isa.context().sync_status() == isa.ISA_OK
    assert torch.isfinite(out.float()).all()
    res = oracle.attention(qb, kb, vb, off, w.k_block, idx_ref, lw_ref, w.scale, sample)
    o_all = out[0].float().cpu().numpy()
    l_all = lse[0].cpu().numpy()
    g_o, r_o, g_l, r_l = [], [], [], []
    for (_, j, g), (o, l) in zip(sample, res):
        g_o.append(o_all[heads[j], off[g]:off[g + 1]])
        r_o.append(o)
        g_l.append(l_all[heads[j], off[g]:off[g + 1]])
        r_l.append(l)
    g_o = np.concatenate(g_o).astype(np.float64)
    r_o = np.concatenate(r_o)
    assert cases.rel_l2(g_o, r_o) <= cases.ATTN_REL_L2
    assert np.abs(g_o - r_o).max() <= cases.ATTN_MAX_ABS
    assert np.abs(np.concatenate(g_l) - np.concatenate(r_l)).max() < 2e-2
