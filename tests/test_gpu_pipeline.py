"""The fused entry points against the separate ones, on the GPU.

isa_pipeline runs score -> select -> attention inside one call, and
isa_pipeline_host does the same from host buffers in chunks of heads whose
copies overlap the compute.  Both must give exactly what the three separate
calls give, whose parity with the oracle the other GPU tests establish:

  * the plan written by isa_pipeline equals isa_select(isa_score(.)) bit for
    bit (the selector's uniform is keyed by the global head and batch index,
    so chunking must not change it);
  * the outputs equal isa_attention on that plan bit for bit.
Shapes use batch 2 and head counts that do and do not divide into chunks."""
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


@pytest.mark.parametrize("preset,B,H,N,Bk,Bq,ne,ns", [
    ("wan13", 2, 3, 1500, 64, 128, 4, 7),    # one head per chunk
    ("wan13", 1, 10, 1100, 32, 128, 5, 9),   # two heads per chunk, five chunks
    ("tiny", 2, 9, 777, 16, 64, 6, 10),      # two heads per chunk, a last chunk of one
])
def test_pipelines_equal_separate_calls(isa, preset, B, H, N, Bk, Bq, ne, ns):
    ws = [wl.preset(preset, k_block=Bk, q_block=Bq, n_exact=ne, n_sample=ns, seed=s) for s in range(B)]
    ins = [wl.make_inputs(w, "cpu", heads=H, seq_len=N) for w in ws]
    w = ws[0]
    q = torch.cat([i.q for i in ins], 0).contiguous()
    k = torch.cat([i.k for i in ins], 0).contiguous()
    v = torch.cat([i.v for i in ins], 0).contiguous()
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    ctx = isa.context()
    lay = isa.layout_for(qd, Bk, Bq, scale=w.scale)
    p = isa.params(w.n_clusters, w.n_iters, ne, ns, w.seed)
    S = ne + ns

    # separate calls
    mass = isa.score(qd, kd, lay, w.n_clusters, w.n_iters)
    idx, lw = isa.select(mass, lay, ne, ns, w.seed)
    out = isa.attention(qd, kd, vd, idx, lw, lay)
    assert ctx.sync_status() == isa.ISA_OK

    # one device call, plan kept
    pidx = torch.empty(B, H, lay.num_groups, S, dtype=torch.int32, device="cuda")
    plw = torch.empty(B, H, lay.num_groups, S, dtype=torch.float32, device="cuda")
    out_p = isa.pipeline(qd, kd, vd, lay, p, plan_idx=pidx, plan_log_w=plw)
    assert ctx.sync_status() == isa.ISA_OK
    assert torch.equal(pidx, idx)
    assert torch.equal(plw, lw)
    assert torch.equal(out_p, out)

    # from host buffers, chunked by heads with overlapped copies
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    oh = torch.empty_like(q).pin_memory()
    arena = torch.empty(isa.pipeline_host_workspace_bytes(lay, p) + 256, dtype=torch.uint8, device="cuda")
    isa.pipeline_host(qh, kh, vh, oh, lay, p, arena)
    torch.cuda.synchronize()
    assert ctx.sync_status() == isa.ISA_OK
    assert torch.equal(oh, out.cpu())
    # the arena is reused: a second call gives the same bytes
    oh2 = torch.zeros_like(oh).pin_memory()
    isa.pipeline_host(qh, kh, vh, oh2, lay, p, arena)
    torch.cuda.synchronize()
    assert torch.equal(oh2, oh)
