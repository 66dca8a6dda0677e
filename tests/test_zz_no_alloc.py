"""isa_attention_noalloc: attention for callers that cannot allocate.

Some callers have no device memory to lend the library: custom-op or plugin
interfaces that hand a kernel only its inputs and outputs, or latency-critical
code that must not call cudaMalloc.  The no-allocation entry point keeps the
attention kernel's tile-list scratch in an array inside the library.  This
test calls it through the C ABI twice in a row (the second call sees the
array as the first left it) and checks each output, and the log-sum-exp,
against isa_attention with a caller workspace.  Both run the same tile-list
and attention kernels on the same plan, so they must agree bit for bit.  The
case with the longer tile list runs first, so a stale entry left in the array
would show up in the shorter one.  It lives in its own file so that it runs
last."""
import ctypes

import pytest
import torch

from tests import cases
from tests.cases import Case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def isa():
    from block_sparse_importance_b200 import build, isa as m
    build.build()
    return m


def _call_noalloc(isa, q, k, v, idx, lw, out, lse, lay):
    L, ctx = isa.lib(), isa.context()
    sh = lay.c()
    st = L.isa_attention_noalloc(ctx.handle, ctypes.byref(sh), ctypes.c_void_p(q.data_ptr()),
                                 ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
                                 ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(lw.data_ptr()),
                                 int(idx.shape[-1]), ctypes.c_void_p(out.data_ptr()),
                                 ctypes.c_void_p(lse.data_ptr()),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == isa.ISA_OK, L.isa_last_error(ctx.handle).decode()


def test_noalloc_matches_workspace_call_twice(isa):
    runs = [
        Case("wan13", 2, 3000, 32, 200, 3, 5),    # uniform groups above one tile: 30 tiles
        Case("wan13", 2, 1500, 64, 128, 4, 6, offsets=cases.random_offsets(1500, 16, 300, seed=11)),
    ]
    for c in runs:
        q, k, v = c.cuda()
        idx, lw = [torch.from_numpy(t).cuda() for t in c.plan()]
        lay = c.layout()
        ref, ref_lse = isa.attention(q, k, v, idx, lw, lay, want_lse=True)
        assert isa.context().sync_status() == isa.ISA_OK
        for _ in range(2):
            out = torch.full_like(q, float("nan"))
            lse = torch.full(q.shape[:-1], float("nan"), dtype=torch.float32, device=q.device)
            _call_noalloc(isa, q, k, v, idx, lw, out, lse, lay)
            assert isa.context().sync_status() == isa.ISA_OK
            assert torch.equal(out, ref)
            assert torch.equal(lse, ref_lse)


def test_noalloc_rejects_shapes_beyond_its_scratch(isa):
    lay = isa.Layout(1, 1, 4_000_000, 128, 16, 64, 250_000, 0.088,
                     q_offsets=torch.zeros(250_001, dtype=torch.int32, device="cuda"))
    L, ctx = isa.lib(), isa.context()
    sh = lay.c()
    t = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    st = L.isa_attention_noalloc(ctx.handle, ctypes.byref(sh), ctypes.c_void_p(t.data_ptr()),
                                 ctypes.c_void_p(t.data_ptr()), ctypes.c_void_p(t.data_ptr()),
                                 ctypes.c_void_p(t.data_ptr()), ctypes.c_void_p(t.data_ptr()), 1,
                                 ctypes.c_void_p(t.data_ptr()), None, None)
    assert st == isa.ISA_ERR_INVALID_ARG
    assert "scratch" in L.isa_last_error(ctx.handle).decode()
