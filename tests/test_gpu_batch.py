"""GPU parity at batch 2: every entry point flattens (batch, head) and the
selector's uniform is keyed by the batch index too (Philox counter
(g, h, b, 0)), so a second batch entry must select and attend on its own.

  * scorer: GPU mass of both entries within relative L2 1e-3 of the oracle
    (groups without a k-means near tie);
  * selector: the oracle's mass fed to both selectors; block indices
    bit-exact and log-weights within 1e-6;
  * attention: the oracle's plan fed to both; within relative L2 1e-2 and
    max abs 2e-2, and the two entries differ (different inputs, different
    uniforms)."""
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


@pytest.mark.parametrize("preset,N,Bk,Bq,ne,ns", [
    ("wan13", 1500, 64, 128, 4, 7),
    ("tiny", 777, 16, 64, 6, 10),
])
def test_batch_two_matches_oracle(isa, preset, N, Bk, Bq, ne, ns):
    H = 2
    ws = [wl.preset(preset, k_block=Bk, q_block=Bq, n_exact=ne, n_sample=ns, seed=s) for s in (0, 1)]
    ins = [wl.make_inputs(w, "cpu", heads=H, seq_len=N) for w in ws]
    w = ws[0]
    q = torch.cat([i.q for i in ins], 0)  # [2, H, N, d]
    k = torch.cat([i.k for i in ins], 0)
    v = torch.cat([i.v for i in ins], 0)
    off = ins[0].offsets
    qb, kb, vb = (wl.bf16_bits(t) for t in (q, k, v))
    G = len(off) - 1
    ctx = isa.context()
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    lay = isa.layout_for(qd, Bk, Bq, scale=w.scale)

    # scorer
    mass = isa.score(qd, kd, lay, w.n_clusters, w.n_iters)
    assert ctx.sync_status() == isa.ISA_OK
    m_ref, _, _, amb = oracle.score(qb, kb, off, Bk, w.n_clusters, w.n_iters, w.scale)
    ok = ~amb.astype(bool)
    assert ok.mean() >= 0.85
    r = cases.rel_l2(mass.cpu().numpy()[ok], m_ref[ok])
    assert r <= cases.MASS_REL_L2, r

    # selector on the oracle's mass (the seed is shared; the uniform differs by b)
    m32 = m_ref.astype(np.float32)
    idx_ref, lw_ref, bad = oracle.select(m32, ne, ns, w.seed)
    assert not bad
    idx, lw = isa.select(torch.from_numpy(m32).cuda(), lay, ne, ns, w.seed)
    assert ctx.sync_status() == isa.ISA_OK
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    assert np.max(np.abs(lw.cpu().numpy() - lw_ref)) <= cases.LOGW_ABS

    # attention on the oracle's plan
    out, lse = isa.attention(qd, kd, vd, torch.from_numpy(idx_ref).cuda(), torch.from_numpy(lw_ref).cuda(), lay,
                             want_lse=True)
    assert ctx.sync_status() == isa.ISA_OK
    groups = [(b, h, g) for b in range(2) for h in range(H) for g in range(G)]
    res = oracle.attention(qb, kb, vb, off, Bk, idx_ref, lw_ref, w.scale, groups)
    ref = np.zeros((2, H, N, w.head_dim))
    ref_lse = np.zeros((2, H, N))
    for (b, h, g), (o, l) in zip(groups, res):
        ref[b, h, off[g]:off[g + 1]] = o
        ref_lse[b, h, off[g]:off[g + 1]] = l
    cases.check_attention(out, ref, lse, ref_lse)
    o = out.float().cpu().numpy()
    assert not np.allclose(o[0], o[1])
