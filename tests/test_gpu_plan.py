"""isa_plan (score -> select in one call, the mass kept in L2 in chunks of
heads) gives the plan isa_select(isa_score(.)) gives, bit for bit, at the
full layer sizes of the presets and with a batch of two."""
import numpy as np
import pytest
import torch

from block_sparse_importance_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def isa():
    from block_sparse_importance_b200 import build, isa as m
    build.build()
    return m


@pytest.mark.parametrize("name", ["tiny", "wan13", "wan14_10", "hunyuan", "varclust"])
def test_plan_equals_score_then_select(isa, name):
    w = wl.preset(name)
    inp = wl.make_inputs(w, "cuda")
    off = torch.from_numpy(inp.offsets).cuda() if w.variable_groups else None
    lay = isa.layout_for(inp.q, w.k_block, w.q_block, q_offsets=off, scale=w.scale)
    p = isa.params(w.n_clusters, w.n_iters, w.n_exact, w.n_sample, w.seed)
    mass = isa.score(inp.q, inp.k, lay, w.n_clusters, w.n_iters)
    idx_ref, lw_ref = isa.select(mass, lay, w.n_exact, w.n_sample, w.seed)
    del mass
    idx, lw = isa.plan(inp.q, inp.k, lay, p)
    assert isa.context().sync_status() == isa.ISA_OK
    assert torch.equal(idx, idx_ref)
    assert torch.equal(lw, lw_ref)
    # the workspace holds one chunk's scratch and mass: less than the separate
    # calls need (the whole layer's scorer scratch and mass tensor)
    B, H, N, d = inp.q.shape
    separate = isa.score_workspace_bytes(lay, w.n_clusters) + B * H * lay.num_groups * lay.n_key_blocks * 4
    assert isa.plan_workspace_bytes(lay, p) <= separate


def test_plan_batch_two(isa):
    ws = [wl.preset("wan13", seed=s) for s in (0, 1)]
    ins = [wl.make_inputs(w, "cuda", heads=5, seq_len=4000) for w in ws]
    q = torch.cat([i.q for i in ins], 0).contiguous()
    k = torch.cat([i.k for i in ins], 0).contiguous()
    w = ws[0]
    lay = isa.layout_for(q, w.k_block, w.q_block, scale=w.scale)
    p = isa.params(w.n_clusters, w.n_iters, w.n_exact, w.n_sample, 7)
    mass = isa.score(q, k, lay, w.n_clusters, w.n_iters)
    idx_ref, lw_ref = isa.select(mass, lay, w.n_exact, w.n_sample, 7)
    idx, lw = isa.plan(q, k, lay, p)
    assert isa.context().sync_status() == isa.ISA_OK
    assert torch.equal(idx, idx_ref) and torch.equal(lw, lw_ref)
