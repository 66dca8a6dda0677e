"""GPU parity of the token clustering (the permuted layout of permuted
block-sparse attention; "InstaGen", abstract) against the oracle, step by
step on seeded inputs, and of the permuted attention flow against the
unpermuted one:

  * assign: labels equal the oracle's for the same fp32 centroids, except
    rows the oracle flags as near ties, whose label must be within the tie
    margin of the best;
  * sort: perm, offsets and the non-empty groups equal the oracle's stable
    counting sort of the same labels, bit for bit;
  * update: centroids within fp32 summation error of the oracle's means;
  * the whole clustering: on every head the oracle clusters without a near
    tie, labels, perm and offsets equal the oracle's and the centroids agree
    to fp32 accuracy; on the others the layout is valid;
  * permute_rows: a gather equals indexing, a scatter undoes it;
  * the permuted flow: dense attention on clustered-and-permuted tensors,
    un-permuted, equals dense attention on the originals; and the sparse
    path on the permuted layout with every key block in the plan (one
    query group per non-empty query cluster) equals it too."""
import numpy as np
import pytest
import torch

import oracle
from tests import cases
from block_sparse_importance_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def isa():
    from block_sparse_importance_b200 import build, isa as m
    build.build()
    return m


def _inputs(preset, H, N):
    w = wl.preset(preset)
    return wl.make_inputs(w, "cpu", heads=H, seq_len=N), w


def _f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("preset,H,N,C", [("wan13", 2, 1000, 37), ("wan13", 1, 777, 130), ("tiny", 2, 1500, 64)])
def test_assign_matches_oracle(isa, preset, H, N, C):
    inp, _ = _inputs(preset, H, N)
    x = inp.q
    xb = wl.bf16_bits(x)
    rng = np.random.default_rng(N + C)
    d = x.shape[-1]
    rows = rng.integers(0, N, (1, H, C))
    mu = np.take_along_axis(_f64(xb), rows[..., None], axis=2) + rng.normal(0.0, 0.1, (1, H, C, d))
    mu = mu.astype(np.float32)
    lab = isa.cluster_assign(x.cuda(), torch.from_numpy(mu).cuda())
    assert isa.context().sync_status() == isa.ISA_OK
    lab = lab.cpu().numpy()
    for h in range(H):
        ref, amb = oracle.cluster_assign(xb[0, h], mu[0, h].astype(np.float64))
        ok = ~amb
        assert np.array_equal(lab[0, h][ok], ref[ok])
        if amb.any():
            xr = _f64(xb[0, h][amb])
            m = mu[0, h].astype(np.float64)
            dist = ((xr[:, None, :] - m[None]) ** 2).sum(-1)
            got = dist[np.arange(len(xr)), lab[0, h][amb]]
            scale = (xr ** 2).sum(-1) + (m ** 2).sum(-1).max()
            assert np.all(got - dist.min(1) <= oracle.KMEANS_TIE_REL * scale)


@pytest.mark.parametrize("N,C,H", [(5000, 50, 2), (33, 33, 1), (70000, 600, 1), (20000, 8192, 1), (1, 1, 1)])
def test_sort_matches_oracle(isa, N, C, H):
    rng = np.random.default_rng(N)
    lab = rng.integers(0, max(1, C - 3), (1, H, N)).astype(np.int32)  # the top clusters stay empty
    # (the sort splits a head's rows over up to 16 warps: 33 rows leave some warps without rows)
    perm, off, grp, ng = isa.cluster_sort(torch.from_numpy(lab).cuda(), C)
    assert isa.context().sync_status() == isa.ISA_OK
    perm, off, grp, ng = (t.cpu().numpy() for t in (perm, off, grp, ng))
    for h in range(H):
        p_ref, o_ref = oracle.cluster_sort(lab[0, h], C)
        assert np.array_equal(perm[0, h], p_ref)
        assert np.array_equal(off[0, h], o_ref)
        g_ref = np.concatenate([o_ref[:-1][np.diff(o_ref) > 0], [N]])
        assert ng[0, h] == len(g_ref) - 1
        assert np.array_equal(grp[0, h, :len(g_ref)], g_ref)


def test_sort_flags_a_bad_label(isa):
    lab = np.zeros((1, 1, 100), np.int32)
    lab[0, 0, 17] = 9
    isa.cluster_sort(torch.from_numpy(lab).cuda(), 4)
    assert isa.context().sync_status() == isa.ISA_ERR_DEVICE_CHECK


@pytest.mark.parametrize("preset,H,N,C", [("wan13", 2, 1000, 37), ("tiny", 1, 4096, 16)])
def test_update_matches_oracle(isa, preset, H, N, C):
    inp, _ = _inputs(preset, H, N)
    x = inp.k
    xb = wl.bf16_bits(x)
    d = x.shape[-1]
    rng = np.random.default_rng(C)
    lab = rng.integers(0, C - 1, (1, H, N)).astype(np.int32)  # cluster C - 1 is empty
    mu0 = rng.normal(0.0, 1.0, (1, H, C, d)).astype(np.float32)
    perm = np.zeros_like(lab)
    off = np.zeros((1, H, C + 1), np.int32)
    for h in range(H):
        perm[0, h], off[0, h] = oracle.cluster_sort(lab[0, h], C)
    mu = torch.from_numpy(mu0.copy()).cuda()
    isa.cluster_update(x.cuda(), torch.from_numpy(perm).cuda(), torch.from_numpy(off).cuda(), mu)
    assert isa.context().sync_status() == isa.ISA_OK
    mu = mu.cpu().numpy()
    for h in range(H):
        ref, cnt = oracle.cluster_update(xb[0, h], lab[0, h], mu0[0, h].astype(np.float64))
        assert cnt[C - 1] == 0
        assert np.array_equal(mu[0, h, C - 1], mu0[0, h, C - 1])
        np.testing.assert_allclose(mu[0, h], ref, rtol=1e-5, atol=1e-5)


def _valid_layout(lab, perm, off, N, C):
    assert np.array_equal(np.sort(perm), np.arange(N))
    assert np.all(np.diff(lab[perm]) >= 0)
    assert np.array_equal(off, np.concatenate([[0], np.cumsum(np.bincount(lab, minlength=C))]))


@pytest.mark.parametrize("preset,H,N,C,iters", [("tiny", 4, 1024, 16, 3), ("wan13", 3, 1500, 24, 4)])
def test_cluster_matches_oracle(isa, preset, H, N, C, iters):
    inp, _ = _inputs(preset, H, N)
    x = inp.q
    xb = wl.bf16_bits(x)
    r = isa.cluster(x.cuda(), C, iters)
    assert isa.context().sync_status() == isa.ISA_OK
    g = {k: v.cpu().numpy() for k, v in r.items()}
    lab_ref, perm_ref, off_ref, mu_ref, amb = oracle.cluster_tokens(xb, C, iters)
    assert (~amb).sum() >= 1
    for h in range(H):
        _valid_layout(g["labels"][0, h], g["perm"][0, h], g["offsets"][0, h], N, C)
        if amb[0, h]:
            continue
        assert np.array_equal(g["labels"][0, h], lab_ref[0, h])
        assert np.array_equal(g["perm"][0, h], perm_ref[0, h])
        assert np.array_equal(g["offsets"][0, h], off_ref[0, h])
        np.testing.assert_allclose(g["centroids"][0, h], mu_ref[0, h], rtol=1e-5, atol=1e-5)


def test_permute_rows_round_trip(isa):
    inp, _ = _inputs("wan13", 2, 999)
    x = inp.v.cuda()
    rng = np.random.default_rng(3)
    perm = torch.from_numpy(np.stack([rng.permutation(999) for _ in range(2)])[None].astype(np.int32)).cuda()
    y = isa.permute_rows(x, perm)
    back = isa.permute_rows(y, perm, inverse=True)
    assert isa.context().sync_status() == isa.ISA_OK
    idx = perm.long()[..., None].expand(-1, -1, -1, x.shape[-1])
    assert torch.equal(y, torch.gather(x, 2, idx))
    assert torch.equal(back, x)


def test_permuted_flow_matches_unpermuted(isa):
    inp, w = _inputs("wan13", 2, 1536)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    H, N, Bk = q.shape[1], q.shape[2], 64
    rq = isa.cluster(q, 20, 3)
    rk = isa.cluster(k, 20, 3)
    qp = isa.permute_rows(q, rq["perm"])
    kp = isa.permute_rows(k, rk["perm"])
    vp = isa.permute_rows(v, rk["perm"])
    assert isa.context().sync_status() == isa.ISA_OK
    lay = isa.layout_for(q, Bk, 128, scale=w.scale)
    dense = isa.dense_attention(q, k, v, lay)
    dense_p = isa.permute_rows(isa.dense_attention(qp, kp, vp, lay), rq["perm"], inverse=True)
    assert isa.context().sync_status() == isa.ISA_OK
    assert (dense_p.float() - dense.float()).abs().max().item() <= cases.ATTN_MAX_ABS
    # the sparse path per head, one query group per non-empty query cluster,
    # every key block in the plan: the dense limit again
    ng = rq["n_groups"].cpu().numpy()
    nK = -(-N // Bk)
    out_p = torch.empty_like(qp)
    for h in range(H):
        G = int(ng[0, h])
        offs = rq["groups"][0, h, :G + 1].contiguous()
        sl = slice(h, h + 1)
        lay_h = isa.Layout(1, 1, N, q.shape[3], 128, Bk, G, w.scale, offs)
        qh, kh, vh = (t[:, sl].contiguous() for t in (qp, kp, vp))
        mass = isa.score(qh, kh, lay_h, w.n_clusters, w.n_iters)
        idx, lw = isa.select(mass, lay_h, nK, 0, 0)
        out_p[:, sl] = isa.attention(qh, kh, vh, idx, lw, lay_h)
    assert isa.context().sync_status() == isa.ISA_OK
    out = isa.permute_rows(out_p, rq["perm"], inverse=True)
    assert (out.float() - dense.float()).abs().max().item() <= cases.ATTN_MAX_ABS


def test_cluster_arguments(isa):
    # host-side checks: nothing is enqueued
    x = torch.zeros(1, 1, 64, 128, dtype=torch.bfloat16, device="cuda")
    for C, it in [(0, 1), (65, 1), (4, 0)]:
        with pytest.raises(isa.IsaError):
            isa.cluster(x, C, it)
    with pytest.raises(isa.IsaError):
        isa.permute_rows(x, torch.zeros(1, 1, 64, dtype=torch.int32, device="cuda"), out=x)
    assert isa.context().sync_status() == isa.ISA_OK
