"""Threshold selection (Sol-Attn abstract: blocks kept by comparing their proxy
score with a threshold; read as p_ij >= theta, clamped to [kmin, kmax] in
the Top-p order) through the C ABI against the oracle: kept sets equal except
blocks the oracle marks marginal (p within a relative 1e-4 of theta, or
near-ties across a clamped cut), outputs within the bounds."""
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


# theta values chosen for a kept fraction between a few percent and about half
CASES = [
    ("tiny theta 0.05", "tiny", dict(tau=0.05)),
    ("tiny theta 0.1, kmin 2 binds", "tiny", dict(tau=0.1, kmin=2, kmax=4)),
    ("partial tail, d=128 b=128", "tiny", dict(grid=(1, 5, 100), d=128, b=128, H=2, kmax=8, tau=0.05)),
    ("medium theta 0.01", "medium", dict(H=2, tau=0.01)),
    ("medium theta 0.02, no residual", "medium", dict(H=2, tau=0.02, residual=0)),
]


@pytest.mark.parametrize("desc,name,ov", CASES, ids=[c[0] for c in CASES])
def test_threshold_against_oracle(desc, name, ov):
    import block_sparse_attention_33_b200 as sp
    w = get_config(name, **ov)
    Q, K, V = make_qkv(w)
    res = run_library(w, Q, K, V, routing=sp.ROUTING_CENTROID | sp.SELECT_THRESHOLD)
    assert res["status"] == 0
    _ok(oracle_check(w, Q, K, V, res, selection="threshold"))


def test_threshold_with_pama_and_hilbert_permutation():
    import block_sparse_attention_33_b200 as sp
    w = get_config("stress", H=2, tau=0.005)
    Q, K, V = make_qkv(w)
    perm = sp.spattn_hilbert_perm(*w.grid)
    res = run_library(w, Q, K, V, perm=perm, routing=sp.ROUTING_PAMA | sp.SELECT_THRESHOLD)
    assert res["status"] == 0
    rows = {(0, h): perm[np.arange(0, w.N, 97)] for h in range(w.H)}
    _ok(oracle_check(w, Q, K, V, res, perm=perm, rows=rows, routing="pama", selection="threshold"))


def test_threshold_zero_keeps_everything_like_tau_one():
    """theta = 0 keeps every block, as tau = 1 does under Top-p: same CSR and
    bit-identical output."""
    import block_sparse_attention_33_b200 as sp
    w = get_config("medium", H=2)
    Q, K, V = make_qkv(w)
    a = run_library(w, Q, K, V, routing=sp.ROUTING_CENTROID | sp.SELECT_THRESHOLD, tau=0.0)
    c = run_library(w, Q, K, V, routing=sp.ROUTING_CENTROID, tau=1.0)
    assert np.array_equal(a["row_ptr"], c["row_ptr"]) and np.array_equal(a["col_idx"], c["col_idx"])
    assert a["row_ptr"][-1] == w.H * w.nb * w.nb
    assert np.array_equal(a["O"], c["O"])


@pytest.mark.parametrize("theta,kmax", [(0.005, 256), (0.002, 64)],
                         ids=["wan theta 0.005 (no clamp)", "wan theta 0.002, kmax 64 (every row clamped)"])
def test_threshold_at_wan_size(theta, kmax):
    """nb = 256: above 128 blocks a binding clamp takes the binary-search
    top-k; routing is compared on every query block, outputs on the sampled
    rows of the full-size tests."""
    import block_sparse_attention_33_b200 as sp
    from tests.test_gpu_full_size import sample_rows
    w = get_config("wan", H=2, tau=theta, kmax=kmax)
    Q, K, V = make_qkv(w)
    res = run_library(w, Q, K, V, routing=sp.ROUTING_CENTROID | sp.SELECT_THRESHOLD)
    assert res["status"] == 0
    rows = sample_rows(w, res, None)
    _ok(oracle_check(w, Q, K, V, res, rows=rows, selection="threshold"))
