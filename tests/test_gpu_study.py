"""The estimator study (IS against truncation and against the unweighted
sample, at a fixed budget, relative to the dense limit).

test_estimator_study_small: the study runs end to end on a small layer;
every plan's error is finite, and with clustered values a larger budget
brings every plan closer to the dense output.

test_estimator_study_matches_oracle: the figures the study reports are the
figures the fp64 oracle gets.  The oracle recomputes the dense output and
each plan's sparse output from the same bf16 tensors and the study's own
plans, and its relative L2 errors must equal the study's within 1e-2."""
import math

import numpy as np
import pytest

import oracle
from block_sparse_importance_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def test_estimator_study_small():
    from block_sparse_importance_b200 import build
    build.build()
    from block_sparse_importance_b200 import estimator_study as st
    lo = st.run("tiny", heads=1, temps=(1.0,), seeds=(0, 1), density=0.1, values="clustered")
    hi = st.run("tiny", heads=1, temps=(1.0,), seeds=(0, 1), density=0.5, values="clustered")
    assert lo["status"] == 0 and hi["status"] == 0
    for res in (lo, hi):
        for r in res["rows"]:
            for key in ("is", "top_s", "unweighted", "is_small_blk"):
                assert math.isfinite(r[key]) and r[key] >= 0.0
    for key in ("is", "top_s", "unweighted"):
        assert hi["rows"][0][key] < lo["rows"][0][key]


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def test_estimator_study_matches_oracle():
    from block_sparse_importance_b200 import build
    build.build()
    from block_sparse_importance_b200 import estimator_study as st
    res = st.run("tiny", heads=1, temps=(0.5, 2.0), seeds=(0, 1), density=0.1, values="clustered",
                 keep_plans=True)
    assert res["status"] == 0
    q, k, v = (wl.bf16_bits(t) for t in res["qkv"])
    B, H, N, d = q.shape
    off = np.asarray(res["offsets"], np.int32)
    G = len(off) - 1
    for row in res["rows"]:
        scale = row["t"] / math.sqrt(d)
        dense, _ = oracle.dense_attention(q, k, v, scale, [(h, r) for h in range(H) for r in range(N)])
        dense = dense.reshape(H, N, d)

        def sparse(idx, lw, bk):
            out = np.zeros((H, N, d))
            got = oracle.attention(q, k, v, off, bk, idx.numpy(), lw.numpy(), scale,
                                   [(0, h, g) for h in range(H) for g in range(G)])
            i = 0
            for h in range(H):
                for g in range(G):
                    out[h, off[g]:off[g + 1]] = got[i][0]
                    i += 1
            return out

        for name in ("is", "unweighted", "top_s", "is_small_blk"):
            errs = [_rel(sparse(idx, lw, bk), dense) for idx, lw, bk in row["plans"][name]]
            ref = sum(errs) / len(errs)
            assert abs(ref - row[name]) <= 1e-2, (row["t"], name, ref, row[name])
