"""Pins of the oracle's sparse and dense attention: the dense limit against a
library attention (torch scaled_dot_product_attention in fp64 on CPU), the
sparse pass against the same library routine with an additive mask that
keeps only the plan's key rows and carries the log-weights, and the
log-weight shift against block duplication (ln 2 shift == the block twice)."""
import math

import numpy as np
import torch
import torch.nn.functional as F

import oracle
from block_sparse_importance_b200 import workloads as wl


def _f64(bits):
    return torch.from_numpy((bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64))


def _inputs(H=2, N=300, d=32, seed=0):
    g = torch.Generator().manual_seed(seed)
    q, k, v = [torch.randn(1, H, N, d, generator=g).to(torch.bfloat16) for _ in range(3)]
    return [wl.bf16_bits(t) for t in (q, k, v)]


def _sdpa(q, k, v, scale, mask=None):
    return F.scaled_dot_product_attention(_f64(q), _f64(k), _f64(v), attn_mask=mask, scale=scale)


def test_dense_limit_matches_library_attention():
    q, k, v = _inputs()
    N, d, H = 300, 32, 2
    scale = 1 / math.sqrt(d)
    ref = _sdpa(q, k, v, scale)[0]
    rows = [(h, r) for h in range(H) for r in range(0, N, 7)]
    out, lse = oracle.dense_attention(q, k, v, scale, rows)
    want = np.stack([ref[h, r].numpy() for h, r in rows])
    assert np.max(np.abs(out - want)) < 1e-12
    # all blocks exact, log_w = 0: the sparse pass is dense attention, with a
    # partial last key block (16) and with blocks that divide N (20)
    for Bk in (16, 20):
        Bq = 64
        off = np.minimum(np.arange(0, N + Bq, Bq), N).astype(np.int32)
        G, nK = len(off) - 1, -(-N // Bk)
        idx = np.tile(np.arange(nK, dtype=np.int32), (1, H, G, 1))
        lw = np.zeros_like(idx, dtype=np.float32)
        res = oracle.attention(q, k, v, off, Bk, idx, lw, scale, [(0, h, g) for h in range(H) for g in range(G)])
        i = 0
        for h in range(H):
            for g in range(G):
                o, l = res[i]
                i += 1
                assert np.max(np.abs(o - ref[h, off[g]:off[g + 1]].numpy())) < 1e-12


def test_sparse_pass_matches_masked_library_attention():
    q, k, v = _inputs(seed=1)
    N, d, H, Bk, Bq = 300, 32, 2, 16, 64
    scale = 1 / math.sqrt(d)
    off = np.minimum(np.arange(0, N + Bq, Bq), N).astype(np.int32)
    G, nK = len(off) - 1, -(-N // Bk)
    rng = np.random.default_rng(0)
    S = 6
    idx = np.zeros((1, H, G, S), np.int32)
    lw = (rng.random((1, H, G, S)) * 3).astype(np.float32)
    for h in range(H):
        for g in range(G):
            if g == 0:   # include the partial tail block (300 = 18*16 + 12)
                idx[0, h, g] = np.sort(np.append(rng.choice(nK - 1, S - 1, replace=False), nK - 1))
            else:
                idx[0, h, g] = np.sort(rng.choice(nK, S, replace=False))
    groups = [(0, h, g) for h in range(H) for g in range(G)]
    res = oracle.attention(q, k, v, off, Bk, idx, lw, scale, groups)
    i = 0
    for h in range(H):
        for g in range(G):
            bias = torch.full((N,), -math.inf, dtype=torch.float64)
            for s in range(S):
                b = idx[0, h, g, s]
                bias[b * Bk:min(N, (b + 1) * Bk)] = float(lw[0, h, g, s])
            ref = _sdpa(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1], scale, bias.view(1, 1, 1, N))[0, 0]
            o, l = res[i]
            i += 1
            assert np.max(np.abs(o - ref[off[g]:off[g + 1]].numpy())) < 1e-12
            # lse = log of the weighted softmax denominator
            z = scale * _f64(q[0, h, off[g]:off[g + 1]]) @ _f64(k[0, h]).T + bias
            assert np.max(np.abs(l - torch.logsumexp(z, dim=-1).numpy())) < 1e-10


def test_log_weight_shift_equals_block_duplication():
    q, k, v = _inputs(H=1, N=128, d=16, seed=2)
    scale = 0.25
    off = np.array([0, 64, 128], np.int32)
    idx2 = np.array([[[[0, 3, 5], [1, 2, 6]]]], np.int32)
    lw2 = np.array([[[[0.0, math.log(2.0), 0.0], [0.0, 0.0, math.log(2.0)]]]], np.float32)
    idx_dup = np.array([[[[0, 3, 3, 5], [1, 2, 6, 6]]]], np.int32)
    lw_dup = np.zeros_like(idx_dup, dtype=np.float32)
    a = oracle.attention(q, k, v, off, 16, idx2, lw2, scale, [(0, 0, 0), (0, 0, 1)])
    b = oracle.attention(q, k, v, off, 16, idx_dup, lw_dup, scale, [(0, 0, 0), (0, 0, 1)])
    for (oa, la), (ob, lb) in zip(a, b):
        assert np.max(np.abs(oa - ob)) < 1e-7 and np.max(np.abs(la - lb)) < 1e-7


def test_variable_groups_use_their_own_rows():
    q, k, v = _inputs(H=1, N=200, d=16, seed=3)
    off = np.array([0, 17, 150, 200], np.int32)
    idx = np.tile(np.arange(4, dtype=np.int32), (1, 1, 3, 1))
    idx[0, 0, 1] = [0, 4, 8, 12]
    lw = np.zeros_like(idx, dtype=np.float32)
    res = oracle.attention(q, k, v, off, 16, idx, lw, 0.3, [(0, 0, 1)])
    (o, l), = res
    assert o.shape == (133, 16)
    keys = np.concatenate([np.arange(b * 16, min(200, b * 16 + 16)) for b in [0, 4, 8, 12]])
    ref = _sdpa(q[:, :, 17:150], k[:, :, keys], v[:, :, keys], 0.3)[0, 0].numpy()
    assert np.max(np.abs(o - ref)) < 1e-12
