"""PAMA routing (per-query softmax over key-block centroids, averaged per
query block; PARK page 5.1) through the C ABI against the oracle: kept sets
equal except blocks the oracle marks marginal, outputs within the bounds."""
import numpy as np
import pytest

from tests.harness import MAX_ABS, REL_L2, oracle_check, run_library
from workloads import get_config, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu(gpu_required):
    import block_sparse_attention_33_b200 as sp
    sp.lib()


def _ok(fig):
    assert fig["bad"] == 0, fig
    assert fig["max_abs"] < MAX_ABS and fig["rel_l2"] < REL_L2, fig


CASES = [
    ("tiny (d=64, b=64)", "tiny", dict()),
    ("tiny tau 0.6, kmax 4", "tiny", dict(tau=0.6, kmax=4)),
    ("partial tail, d=128 b=128", "tiny", dict(grid=(1, 5, 100), d=128, b=128, H=2, kmax=8, tau=0.8)),
    ("medium, 2 heads", "medium", dict(H=2)),
    ("medium, no residual", "medium", dict(H=2, residual=0, tau=0.8)),
]


@pytest.mark.parametrize("desc,name,ov", CASES, ids=[c[0] for c in CASES])
def test_pama_against_oracle(desc, name, ov):
    import block_sparse_attention_33_b200 as sp
    w = get_config(name, **ov)
    Q, K, V = make_qkv(w)
    res = run_library(w, Q, K, V, routing=sp.ROUTING_PAMA)
    assert res["status"] == 0
    _ok(oracle_check(w, Q, K, V, res, routing="pama"))


def test_pama_with_hilbert_permutation():
    import block_sparse_attention_33_b200 as sp
    w = get_config("stress", H=2)
    Q, K, V = make_qkv(w)
    perm = sp.spattn_hilbert_perm(*w.grid)
    res = run_library(w, Q, K, V, perm=perm, routing=sp.ROUTING_PAMA)
    assert res["status"] == 0
    rows = {(0, h): perm[np.arange(0, w.N, 97)] for h in range(w.H)}
    _ok(oracle_check(w, Q, K, V, res, perm=perm, rows=rows, routing="pama"))


def test_pama_and_centroid_routings_differ_and_tau_one_is_dense():
    """The two estimates pick different sets on the medium layer; at tau = 1
    both keep everything and give the same output."""
    import block_sparse_attention_33_b200 as sp
    w = get_config("medium", H=2)
    Q, K, V = make_qkv(w)
    a = run_library(w, Q, K, V, routing=sp.ROUTING_PAMA)
    c = run_library(w, Q, K, V, routing=sp.ROUTING_CENTROID)
    assert not (np.array_equal(a["row_ptr"], c["row_ptr"]) and np.array_equal(a["col_idx"], c["col_idx"]))
    a1 = run_library(w, Q, K, V, routing=sp.ROUTING_PAMA, tau=1.0)
    c1 = run_library(w, Q, K, V, routing=sp.ROUTING_CENTROID, tau=1.0)
    assert np.array_equal(a1["O"], c1["O"])
