"""The tcgen05/TMEM attention kernel (128-token blocks) against the oracle and
against the independent warp-MMA kernel on the same inputs and CSR."""
import os

import numpy as np
import pytest

from tests.harness import MAX_ABS, REL_L2, compare_outputs, oracle_check, run_library
from workloads import get_config, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu(gpu_required):
    import block_sparse_attention_33_b200 as sp
    sp.lib()


def run_with(kernel, w, Q, K, V, **kw):
    old = os.environ.get("SPATTN_ATTN")
    try:
        if kernel == "mma":
            os.environ["SPATTN_ATTN"] = "mma"
        else:
            os.environ.pop("SPATTN_ATTN", None)
        return run_library(w, Q, K, V, **kw)
    finally:
        if old is None:
            os.environ.pop("SPATTN_ATTN", None)
        else:
            os.environ["SPATTN_ATTN"] = old


SMALL = [
    ("one block, d=128", dict(grid=(1, 1, 128), d=128, b=128, H=1, kmax=4)),
    ("4 blocks, d=128", dict(grid=(1, 4, 128), d=128, b=128, H=1, kmax=4, tau=0.7)),
    ("partial tail, d=128", dict(grid=(1, 5, 100), d=128, b=128, H=2, kmax=8, tau=0.8)),
    ("d=64 b=128", dict(grid=(2, 8, 64), d=64, b=128, H=2, tau=0.85)),
    ("no residual", dict(grid=(2, 8, 64), d=128, b=128, H=2, tau=0.6, residual=0)),
    ("tau=1 dense", dict(grid=(2, 8, 64), d=128, b=128, H=2, tau=1.0)),
]


@pytest.mark.parametrize("desc,ov", SMALL, ids=[s[0] for s in SMALL])
def test_tc_small_against_oracle_and_mma(desc, ov):
    w = get_config("tiny", **ov)
    Q, K, V = make_qkv(w)
    res = run_with("tc", w, Q, K, V)
    assert res["status"] == 0
    fig = oracle_check(w, Q, K, V, res)
    assert fig["bad"] == 0, fig
    assert fig["max_abs"] < MAX_ABS and fig["rel_l2"] < REL_L2, fig
    ref = run_with("mma", w, Q, K, V)
    assert np.array_equal(ref["row_ptr"], res["row_ptr"])
    max_abs, rel = compare_outputs(res["O"], ref["O"])
    assert max_abs < MAX_ABS and rel < REL_L2, (max_abs, rel)


@pytest.mark.parametrize("residual", [1, 0])
def test_tc_medium(residual):
    w = get_config("medium", residual=residual)
    Q, K, V = make_qkv(w)
    res = run_with("tc", w, Q, K, V)
    assert res["status"] == 0
    fig = oracle_check(w, Q, K, V, res)
    assert fig["bad"] == 0 and fig["max_abs"] < MAX_ABS and fig["rel_l2"] < REL_L2, fig


def test_tc_hilbert_stress_shape_small():
    w = get_config("stress", H=2)
    Q, K, V = make_qkv(w)
    import block_sparse_attention_33_b200 as sp
    perm = sp.spattn_hilbert_perm(*w.grid)
    res = run_with("tc", w, Q, K, V, perm=perm)
    assert res["status"] == 0
    rows = {(0, h): np.arange(0, w.N, 97) for h in range(w.H)}
    fig = oracle_check(w, Q, K, V, res, perm=perm, rows={k: perm[v] for k, v in rows.items()})
    assert fig["bad"] == 0 and fig["max_abs"] < MAX_ABS and fig["rel_l2"] < REL_L2, fig
