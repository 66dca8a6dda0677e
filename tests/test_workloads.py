"""The seeded generators: deterministic, shaped as the presets state."""
import numpy as np
import torch

from block_sparse_importance_b200 import workloads as wl


def test_presets_shapes_and_budgets():
    p = wl.PRESETS
    assert p["tiny"].seq_len == 4096 and p["tiny"].n_key_blocks == 64
    assert (p["wan13"].seq_len, p["wan13"].n_key_blocks, p["wan13"].n_select) == (32760, 512, 51)
    w = p["wan14_10"]
    assert (w.seq_len, w.n_key_blocks, w.n_exact, w.n_sample) == (75600, 1182, 39, 79)
    assert (p["wan14_5"].n_exact, p["wan14_5"].n_sample) == (20, 39)
    assert (p["wan14_20"].n_exact, p["wan14_20"].n_sample) == (79, 157)
    h = p["hunyuan"]
    assert (h.seq_len, h.n_key_blocks, h.n_exact, h.n_sample) == (118800, 7425, 248, 496)
    assert (h.n_select * h.k_block) % 128 == 0


def test_cluster_sizes():
    s = wl.cluster_sizes(600, 75600, 0)
    assert s.sum() == 75600 and s.min() >= 16 and s.max() <= 1024 and len(s) == 600
    off = wl.group_offsets(wl.PRESETS["varclust"])
    assert off[0] == 0 and off[-1] == 75600 and np.all(np.diff(off) >= 16)


def test_inputs_deterministic_and_clustered():
    w = wl.preset("tiny")
    a = wl.make_inputs(w, "cpu")
    b = wl.make_inputs(w, "cpu")
    assert a.q.dtype == torch.bfloat16 and a.q.shape == (1, 1, 4096, 64)
    assert torch.equal(a.q, b.q) and torch.equal(a.k, b.k) and torch.equal(a.v, b.v)
    assert list(a.offsets[:3]) == [0, 64, 128] and a.offsets[-1] == 4096
    # tokens of one 8x8 cell share a centre: their queries correlate strongly
    q = a.q[0, 0].float()
    same = torch.nn.functional.cosine_similarity(q[0], q[1], dim=0)
    assert same > 0.5
    t = wl.make_inputs(w, "cpu", seq_len=1000)
    assert t.q.shape[2] == 1000 and t.offsets[-1] == 1000
