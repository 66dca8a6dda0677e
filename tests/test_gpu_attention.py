"""GPU parity of isa_attention / isa_dense_attention against the fp64 oracle
(plans made by the oracle), through the C-ABI, on cases that span several
tiles, ragged group / key tails, every key-block size, uniform groups below
and above one tile, and variable clusters."""
import math

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


def _run_sparse(isa, c: Case):
    idx, lw = c.plan()
    q, k, v = c.cuda()
    lay = c.layout()
    out, lse = isa.attention(q, k, v, torch.from_numpy(idx).cuda(), torch.from_numpy(lw).cuda(), lay,
                             want_lse=True)
    assert isa.context().sync_status() == isa.ISA_OK
    ref, ref_lse = c.oracle_attention()
    return cases.check_attention(out, ref, lse, ref_lse)


@pytest.mark.parametrize("d_preset,N,Bk,Bq,ne,ns", [
    ("tiny", 1000, 64, 64, 4, 4),        # d=64, 64-row groups, ragged tails
    ("wan13", 1500, 64, 128, 4, 7),      # odd block count: half-empty last KV tile
    ("wan13", 1200, 16, 128, 8, 16),     # 16-row sub-blocks gathered into tiles
    ("wan13", 1000, 32, 96, 5, 6),
    ("wan13", 1000, 128, 128, 2, 3),
    ("wan13", 1000, 64, 200, 3, 5),      # groups larger than a tile (tile list)
    ("tiny", 777, 16, 128, 6, 10),
])
def test_sparse_matches_oracle(isa, d_preset, N, Bk, Bq, ne, ns):
    c = Case(d_preset, 2, N, Bk, Bq, ne, ns)
    _run_sparse(isa, c)


def test_variable_clusters_match_oracle(isa):
    off = cases.random_offsets(1500, 16, 300, seed=3)
    c = Case("wan13", 2, 1500, 64, 128, 4, 6, offsets=off)
    _run_sparse(isa, c)


def test_full_plan_equals_dense(isa):
    c = Case("wan13", 2, 700, 64, 128, 11, 0)   # nK = 11: every block exact
    q, k, v = c.cuda()
    lay = c.layout()
    idx, lw = c.plan()
    assert np.all(np.sort(idx, axis=-1) == np.arange(11))
    sparse = isa.attention(q, k, v, torch.from_numpy(idx).cuda(), torch.from_numpy(lw).cuda(), lay)
    dense = isa.dense_attention(q, k, v, lay)
    torch.cuda.synchronize()
    assert (sparse.float() - dense.float()).abs().max().item() < 2e-3


@pytest.mark.parametrize("preset,N,H", [("tiny", 1000, 2), ("wan13", 1000, 2), ("wan13", 2048, 1), ("tiny", 50, 1)])
def test_dense_matches_oracle(isa, preset, N, H):
    c = Case(preset, H, N, 64, 128, 1, 0)
    q, k, v = c.cuda()
    lay = c.layout()
    out, lse = isa.dense_attention(q, k, v, lay, want_lse=True)
    assert isa.context().sync_status() == isa.ISA_OK
    rows = [(h, r) for h in range(H) for r in range(N)]
    qb, kb, vb = c.bits
    ref, ref_lse = oracle.dense_attention(qb, kb, vb, c.w.scale, rows)
    o = out.float().cpu().numpy().reshape(H * N, -1)
    assert np.abs(o - ref).max() <= cases.DENSE_MAX_ABS
    assert np.abs(lse.cpu().numpy().reshape(-1) - ref_lse).max() < 1e-2


def test_out_of_range_index_is_reported_not_faulted(isa):
    c = Case("wan13", 1, 600, 64, 128, 2, 2)
    idx, lw = c.plan()
    idx = idx.copy()
    idx[0, 0, 1, 1] = 10_000
    q, k, v = c.cuda()
    out = isa.attention(q, k, v, torch.from_numpy(idx).cuda(), torch.from_numpy(lw).cuda(), c.layout())
    assert isa.context().sync_status() == isa.ISA_ERR_DEVICE_CHECK
    assert torch.isfinite(out.float()).all()
    assert isa.context().sync_status() == isa.ISA_OK   # the word was cleared


def test_host_checks_reject_bad_arguments(isa):
    c = Case("wan13", 1, 600, 64, 128, 2, 2)
    q, k, v = c.cuda()
    idx, lw = [torch.from_numpy(t).cuda() for t in c.plan()]
    lay = c.layout()
    import ctypes
    L, ctx = isa.lib(), isa.context()
    sh = lay.c()
    st = L.isa_attention(ctx.handle, ctypes.byref(sh), ctypes.c_void_p(q.data_ptr() + 2), ctypes.c_void_p(k.data_ptr()),
                         ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(idx.data_ptr()),
                         ctypes.c_void_p(lw.data_ptr()), 4, ctypes.c_void_p(q.data_ptr()), None, None, 0, None)
    assert st == isa.ISA_ERR_INVALID_ARG                      # q not 16-byte aligned
    assert "aligned" in L.isa_last_error(ctx.handle).decode()
    bad = c.layout()
    bad.head_dim = 96
    with pytest.raises(isa.IsaError) as e:
        isa.dense_attention(q, k, v, bad)
    assert e.value.status == isa.ISA_ERR_UNSUPPORTED
    bad = c.layout()
    bad.num_groups = 3
    with pytest.raises(isa.IsaError):
        isa.attention(q, k, v, idx, lw, bad)


@pytest.mark.parametrize("Bk,ne,ns", [(64, 4, 7), (16, 8, 16)])
def test_logit_jumps_match_oracle(isa, Bk, ne, ns):
    """Plans whose later blocks carry log-weights far above the earlier ones
    (jumps of 30, 50 and 100 nats, i.e. 43, 72 and 144 log2 units, at the last
    or a middle plan position) and far below (-100): the running max must be
    raised, P rescaled and O kept finite on every such path."""
    c = Case("wan13", 2, 1200, Bk, 128, ne, ns)
    idx, lw = c.plan()
    lw = lw.copy()
    S = lw.shape[-1]
    jumps = [(S - 1, 30.0), (S - 1, 50.0), (S - 1, 100.0), (S // 2, 60.0), (S // 2, -100.0), (0, 0.0)]
    for h in range(c.H):
        for g in range(c.G):
            pos, add = jumps[(h * c.G + g) % len(jumps)]
            lw[0, h, g, pos] += add
    q, k, v = c.cuda()
    out, lse = isa.attention(q, k, v, torch.from_numpy(idx).cuda(), torch.from_numpy(lw).cuda(), c.layout(),
                             want_lse=True)
    assert isa.context().sync_status() == isa.ISA_OK
    ref, ref_lse = c.oracle_attention(idx, lw)
    cases.check_attention(out, ref, lse, ref_lse)
