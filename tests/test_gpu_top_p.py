"""GPU parity of isa_select_top_p (exact-set size set by a share p of each
row's mass, "iCATS" top-p sparsity; the rest of the budget sampled) against
the oracle fed the identical fp32 mass: per-row exact-set sizes and block
indices bit-exact, log-weights within 1e-6.  Rows up to 2048 blocks take
the warp-per-row selector, longer rows the CTA-per-row one; mass kinds with
ties, zeros and a few dominant blocks reach the count's tie rule and its
target-0 case."""
import numpy as np
import pytest
import torch

import oracle
from tests import cases

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def isa():
    from block_sparse_importance_b200 import build, isa as m
    build.build()
    return m


def _mass(kind, rng, H, G, nK):
    if kind == "lognormal":
        m = np.exp(rng.normal(0, 2.0, (1, H, G, nK)))
    elif kind == "ties":
        m = rng.integers(0, 3, (1, H, G, nK)).astype(np.float64)
    elif kind == "spiky":
        m = rng.random((1, H, G, nK)) * 1e-3
        m[..., rng.choice(nK, min(nK, 5), replace=False)] = 100.0
    else:
        m = np.zeros((1, H, G, nK))
        m[0, 0, 0, nK // 2] = 1.0  # one row with a single block, the rest all zero
    return m.astype(np.float32)


@pytest.mark.parametrize("kind", ["lognormal", "ties", "spiky", "zeros"])
@pytest.mark.parametrize("nK,S", [(64, 8), (1182, 118), (300, 1), (2049, 30), (5000, 500)])
@pytest.mark.parametrize("p", [0.1, 0.5, 0.9, 1.0])
def test_select_top_p_bit_exact(isa, kind, nK, S, p):
    rng = np.random.default_rng(nK + S)
    H, G = 2, 6
    mass = _mass(kind, rng, H, G, nK)
    N = nK * 64
    lay = isa.Layout(1, H, N, 128, -(-N // G), 64, G, 0.088)
    assert lay.num_groups == G
    idx_ref, lw_ref, ke_ref, bad = oracle.select_top_p(mass, p, S, 7)
    assert not bad
    idx, lw, ke = isa.select_top_p(torch.from_numpy(mass).cuda(), lay, p, S, 7)
    assert isa.context().sync_status() == isa.ISA_OK
    assert np.array_equal(ke.cpu().numpy(), ke_ref)
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    assert np.max(np.abs(lw.cpu().numpy() - lw_ref)) <= cases.LOGW_ABS


def test_select_top_p_arguments(isa):
    H, G, nK = 1, 2, 16
    N = nK * 64
    lay = isa.Layout(1, H, N, 128, -(-N // G), 64, G, 0.088)
    m = torch.ones(1, H, G, nK, device="cuda")
    for p, S in [(0.0, 4), (1.5, 4), (0.5, 0), (0.5, nK + 1)]:
        with pytest.raises(isa.IsaError):
            isa.select_top_p(m, lay, p, S, 0)
    assert isa.context().sync_status() == isa.ISA_OK
