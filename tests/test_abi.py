"""The C-ABI library builds, loads without a GPU and exports every entry
point include/isa.h declares; size queries and argument errors behave."""
import ctypes

import pytest

from block_sparse_importance_b200 import build as isa_build
from block_sparse_importance_b200 import isa


@pytest.fixture(scope="module")
def L():
    isa_build.build()
    return isa.lib()


def test_header_declares_the_boundary():
    names = isa.declared_symbols()
    for n in ["isa_create", "isa_destroy", "isa_score", "isa_select", "isa_select_top_p", "isa_attention",
              "isa_dense_attention", "isa_sync_status", "isa_status_string", "isa_score_workspace_bytes",
              "isa_attention_workspace_bytes", "isa_pipeline", "isa_pipeline_host", "isa_cluster",
              "isa_cluster_assign", "isa_cluster_sort", "isa_cluster_update", "isa_cluster_workspace_bytes",
              "isa_permute_rows"]:
        assert n in names


def test_every_declared_symbol_is_exported(L):
    for n in isa.declared_symbols():
        assert hasattr(L, n), n


def test_status_strings(L):
    assert isa.status_string(isa.ISA_OK) == "ok"
    assert "timed out" in isa.status_string(isa.ISA_ERR_TIMEOUT)
    assert isa.status_string(99) == "unknown status"


def test_workspace_sizes(L):
    lay = isa.Layout(1, 40, 75600, 128, 128, 64, 591, 128 ** -0.5)
    nk = 1182
    want = (40 * nk * 128 * 4) + (40 * 591 * 8 * 128 * 4) + (40 * 591 * 8 * 4)
    got = isa.score_workspace_bytes(lay, 8)
    assert want + 4 <= got <= want + 4 * 256                       # + the key-block counter
    assert isa.attention_workspace_bytes(lay) == 0                 # uniform groups need no scratch
    lay.q_block = 200
    lay.num_groups = -(-75600 // 200)
    assert isa.attention_workspace_bytes(lay) >= 16 * (lay.num_groups + 75600 // 128)
    p = isa.params(8, 3, 39, 79, 0)
    assert isa.pipeline_workspace_bytes(lay, p) > got
    assert isa.pipeline_host_workspace_bytes(lay, p) == isa.pipeline_workspace_bytes(lay, p) + 4 * 40 * 75600 * 256


def test_null_context_is_rejected_without_a_device(L):
    sh = isa.Layout(1, 1, 128, 64, 64, 64, 2, 0.125).c()
    st = L.isa_score(None, ctypes.byref(sh), None, None, 4, 3, None, None, None, None, 0, None)
    assert st == isa.ISA_ERR_INVALID_ARG
    st = L.isa_attention(None, ctypes.byref(sh), None, None, None, None, None, 1, None, None, None, 0, None)
    assert st == isa.ISA_ERR_INVALID_ARG
    assert L.isa_sync_status(None, None) == isa.ISA_ERR_INVALID_ARG
    L.isa_destroy(None)


def test_create_fails_cleanly_without_a_gpu(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    h = ctypes.c_void_p()
    assert L.isa_create(0, ctypes.byref(h)) != isa.ISA_OK
    assert not h.value


def test_cluster_workspace_size(L):
    import torch
    x = torch.empty(1, 40, 75600, 128, dtype=torch.bfloat16, device="meta")
    up = lambda n: (n + 255) // 256 * 256  # noqa: E731
    cp = 640  # 600 clusters rounded up to 64
    assert isa.cluster_workspace_bytes(x, 600) == 2 * up(40 * cp * 128 * 2) + up(40 * cp * 4)
    assert isa.cluster_workspace_bytes(x, 0) == 0
