"""Failure detection on the GPU without a fault: a pipeline wait is made to
run out (the MMA warp waits on a barrier that nothing arrives at, with a
50 ms per-wait limit); every CTA takes its abort path, the host reads
ISA_ERR_TIMEOUT from the status word, and the same context then computes a
correct result."""
import numpy as np
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


def test_wait_runs_out_then_context_recovers(isa):
    c = Case("wan13", 2, 1000, 64, 128, 3, 5)
    q, k, v = c.cuda()
    idx, lw = [torch.from_numpy(t).cuda() for t in c.plan()]
    lay = c.layout()
    ctx = isa.Context(0)
    try:
        ctx.debug_set(isa.ISA_DEBUG_WAIT_TIMEOUT_NS, 50_000_000)
        ctx.debug_set(isa.ISA_DEBUG_STALL_ATTENTION, 1)
        isa.attention(q, k, v, idx, lw, lay, ctx=ctx)
        assert ctx.sync_status() == isa.ISA_ERR_TIMEOUT
        assert ctx.sync_status() == isa.ISA_OK            # cleared on read
        ctx.debug_set(isa.ISA_DEBUG_STALL_ATTENTION, 0)
        out = isa.attention(q, k, v, idx, lw, lay, ctx=ctx)
        assert ctx.sync_status() == isa.ISA_OK
        ref, _ = c.oracle_attention()
        cases.check_attention(out, ref)
        with pytest.raises(isa.IsaError):
            ctx.debug_set(99, 1)
    finally:
        ctx.close()
