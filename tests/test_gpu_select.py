"""GPU parity of isa_select against the oracle fed the identical fp32 mass
tensor: block indices bit-exact, log-weights within 1e-6."""
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


def _layout(isa, H, G, nK, Bk=64):
    N = nK * Bk
    return isa.Layout(1, H, N, 128, -(-N // G), Bk, G, 0.088)


def _compare(isa, mass, ne, ns, seed, H, G, nK, Bk=64):
    lay = _layout(isa, H, G, nK, Bk)
    assert lay.num_groups == G
    idx_ref, lw_ref, bad = oracle.select(mass, ne, ns, seed)
    idx, lw = isa.select(torch.from_numpy(mass).cuda(), lay, ne, ns, seed)
    st = isa.context().sync_status()
    idx = idx.cpu().numpy()
    lw = lw.cpu().numpy()
    assert np.array_equal(idx, idx_ref)
    assert np.max(np.abs(lw - lw_ref)) <= cases.LOGW_ABS
    return st, bad


@pytest.mark.parametrize("kind", ["lognormal", "ties", "spiky", "zeros"])
@pytest.mark.parametrize("nK,ne,ns", [(64, 4, 4), (37, 0, 9), (1182, 39, 79), (512, 16, 35), (300, 0, 0 + 1),
                                      (200, 150, 50),
                                      # rows longer than 2048 blocks take the CTA-per-row kernel
                                      (2049, 0, 30), (3000, 40, 80), (7425, 248, 496), (5000, 4990, 5),
                                      (4100, 100, 4000),
                                      # pure top-k (no sample), on both kernels
                                      (64, 8, 0), (3000, 40, 0)])
def test_select_bit_exact(isa, kind, nK, ne, ns):
    rng = np.random.default_rng(nK + ne)
    H, G = 2, 8
    if kind == "lognormal":
        m = np.exp(rng.normal(0, 2.0, (1, H, G, nK)))
    elif kind == "ties":
        m = rng.integers(0, 3, (1, H, G, nK)).astype(np.float64)
    elif kind == "spiky":
        m = rng.random((1, H, G, nK)) * 1e-3
        m[..., rng.choice(nK, min(nK, 5), replace=False)] = 100.0
    else:
        m = np.zeros((1, H, G, nK))
    st, bad = _compare(isa, m.astype(np.float32), ne, ns, 7, H, G, nK)
    assert st == isa.ISA_OK and not bad


def test_select_large_rows_and_seeds(isa):
    rng = np.random.default_rng(1)
    H, G, nK = 2, 6, 7425
    m = np.exp(rng.normal(0, 1.5, (1, H, G, nK))).astype(np.float32)
    for seed in [0, 1, 12345]:
        _compare(isa, m, 248, 496, seed, H, G, nK, Bk=16)


def test_select_on_oracle_mass(isa):
    c = Case("wan13", 2, 3000, 64, 128, 8, 12)
    mass, _, _, _ = c.oracle_mass()
    st, bad = _compare(isa, mass.astype(np.float32), 8, 12, 0, 2, c.G, c.nK)
    assert st == isa.ISA_OK


def test_non_finite_mass_is_flagged(isa):
    H, G, nK = 1, 2, 50
    m = np.ones((1, H, G, nK), np.float32)
    m[0, 0, 1, 3] = np.nan
    st, bad = _compare(isa, m, 2, 4, 3, H, G, nK)
    assert bad and st == isa.ISA_ERR_DEVICE_CHECK
