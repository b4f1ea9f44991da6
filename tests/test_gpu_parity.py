"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Kept-block lists must match the oracle exactly except blocks the oracle marks
marginal (cumulative-mass margin to tau below 1e-4, or a near-tie at the
cut), which are counted.  Outputs must match within max-abs 2e-2 and
relative-L2 4e-3; the oracle attention is evaluated on the library's kept
sets so that an allowed marginal flip does not show up as an output error.
"""
import numpy as np
import pytest

import oracle
from oracle import spattn_ref as R
from tests.harness import (MAX_ABS, REL_L2, compare_outputs, kept_to_csr, oracle_check,
                           run_library, to_dev)
from workloads import Workload, get_config, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu(gpu_required):
    import block_sparse_attention_33_b200 as sp
    sp.lib()


def _assert_ok(fig):
    assert fig["bad"] == 0, fig
    assert fig["max_abs"] < MAX_ABS, fig
    assert fig["rel_l2"] < REL_L2, fig


# ------------------------------------------------------------- pooling ---

@pytest.mark.parametrize("name,overrides", [
    ("tiny", {}), ("medium", {}),
    ("tiny", {"grid": (1, 1, 1000), "b": 128}),        # N % b = 104
    ("tiny", {"grid": (3, 1, 43), "d": 128}),           # N = 129: n_last = 1
])
def test_pool_means_match_oracle(name, overrides):
    w = get_config(name, **overrides)
    Q, K, V = make_qkv(w)
    perm = oracle.hilbert_perm(w.grid) if name == "tiny" and not overrides else None
    res = run_library(w, Q, K, V, perm=perm, want_means=True)
    for X, got in zip((Q, K, V), res["means"]):
        for bi in range(w.B):
            for hi in range(w.H):
                x = R.gather_tokens(R.decode_bf16(X[bi, hi]), perm)
                ref = R.block_means(x, w.b)
                scale = R.block_means(np.abs(x), w.b)
                assert np.all(np.abs(got[bi, hi] - ref) <= 1e-6 * scale + 1e-30)


# ------------------------------------------------------- routing + attn ---

@pytest.mark.parametrize("name,tau,residual", [
    ("tiny", 0.9, 1), ("tiny", 1.0, 1), ("tiny", 0.9, 0),
    ("medium", 0.9, 1), ("medium", 0.9, 0),
])
def test_forward_matches_oracle(name, tau, residual):
    w = get_config(name, tau=tau, residual=residual)
    Q, K, V = make_qkv(w)
    res = run_library(w, Q, K, V)
    assert res["status"] == 0
    fig = oracle_check(w, Q, K, V, res)
    _assert_ok(fig)
    if tau >= 1.0:
        assert fig["kept_fraction"] == 1.0


def test_tau_one_equals_dense_attention():
    w = get_config("tiny", tau=1.0)
    Q, K, V = make_qkv(w)
    res = run_library(w, Q, K, V)
    import torch
    q, k, v = (torch.from_numpy(R.decode_bf16(X)) for X in (Q, K, V))
    dense = torch.nn.functional.scaled_dot_product_attention(q, k, v).numpy()
    max_abs, rel = compare_outputs(res["O"], dense)
    assert max_abs < MAX_ABS and rel < REL_L2


def test_attend_with_oracle_csr_isolates_attention():
    """Attention on the oracle's own kept sets (routing taken out of the loop)."""
    w = get_config("medium", H=2)
    Q, K, V = make_qkv(w)
    ref = R.forward(Q, K, V, w.b, w.tau, w.kmin, w.kmax, w.residual)
    kept = {key: r["kept"] for key, r in ref["route"].items()}
    rp, ci = kept_to_csr(kept, w.B, w.H, w.nb)
    res = run_library(w, Q, K, V, kept_csr=(rp, ci))
    max_abs, rel = compare_outputs(res["O"], ref["O"])
    assert max_abs < MAX_ABS and rel < REL_L2, (max_abs, rel)


def test_hilbert_permuted_forward():
    w = get_config("tiny", tau=0.7, a_scale=2.0, hilbert=True)
    Q, K, V = make_qkv(w)
    import block_sparse_attention_33_b200 as sp
    perm = sp.spattn_hilbert_perm(*w.grid)
    assert np.array_equal(perm, oracle.hilbert_perm(w.grid))
    for residual in (0, 1):
        ww = w.with_(residual=residual)
        res = run_library(ww, Q, K, V, perm=perm)
        _assert_ok(oracle_check(ww, Q, K, V, res, perm=perm))


EDGE = [
    # (description, overrides)
    ("nb=1, N<b", dict(grid=(1, 1, 50), b=64, kmax=4)),
    ("N%b=1", dict(grid=(1, 5, 13), b=64)),               # 65 tokens
    ("N%b=b-1", dict(grid=(1, 1, 191), b=64)),
    ("kmin=kmax", dict(kmin=3, kmax=3)),
    ("kmax>nb", dict(kmax=1000)),
    ("tau<=0", dict(tau=-0.5, kmin=2)),
    ("tau>1", dict(tau=1.5)),
    ("d=128 b=64", dict(d=128, b=64)),
    ("d=64 b=128", dict(b=128)),
    ("B=2", dict(B=2, H=3)),
    ("no residual, kmax=2", dict(residual=0, kmax=2)),
]


@pytest.mark.parametrize("desc,ov", EDGE, ids=[e[0] for e in EDGE])
def test_edge_cases(desc, ov):
    w = get_config("tiny", **ov)
    Q, K, V = make_qkv(w)
    res = run_library(w, Q, K, V)
    assert res["status"] == 0
    fig = oracle_check(w, Q, K, V, res)
    _assert_ok(fig)
    nb = w.nb
    k = np.diff(res["row_ptr"])
    assert np.all(k >= min(w.kmin, nb)) and np.all(k <= min(w.kmax, nb))


def test_random_permutation_and_identity_permutation():
    w = get_config("tiny", tau=0.8)
    Q, K, V = make_qkv(w)
    rng = np.random.default_rng(0)
    for perm in (rng.permutation(w.N), np.arange(w.N)):
        res = run_library(w, Q, K, V, perm=perm)
        _assert_ok(oracle_check(w, Q, K, V, res, perm=perm))


def test_bad_csr_index_is_flagged_not_faulted():
    w = get_config("tiny", H=1)
    Q, K, V = make_qkv(w)
    rp = np.arange(0, w.nb + 1, dtype=np.int32)
    ci = np.full(w.nb, 0, dtype=np.int32)
    ci[3] = w.nb + 5                      # out of range: skipped and flagged
    res = run_library(w, Q, K, V, kept_csr=(rp, ci))
    import block_sparse_attention_33_b200 as sp
    assert res["status"] == sp.ERR_DEVICE


# The same edge cases on 128-token blocks (d = 128), i.e. through the
# persistent tcgen05 attention kernel rather than the warp-MMA one.
EDGE_TC = [
    ("nb=1, N<b", dict(grid=(1, 1, 100))),
    ("N%b=1", dict(grid=(1, 3, 43))),                      # 129 tokens: last block of 1
    ("N%b=b-1", dict(grid=(1, 1, 255))),
    ("kmin=kmax", dict(kmin=3, kmax=3)),
    ("kmax>nb", dict(kmax=1000)),
    ("tau<=0", dict(tau=-0.5, kmin=2)),
    ("tau>1", dict(tau=1.5)),
    ("B=2", dict(B=2, H=3)),
    ("no residual, kmax=2", dict(residual=0, kmax=2)),
    ("d=64", dict(d=64)),
]


@pytest.mark.parametrize("desc,ov", EDGE_TC, ids=[e[0] for e in EDGE_TC])
def test_edge_cases_tcgen05(desc, ov):
    base = dict(grid=(2, 8, 64), d=128, b=128, H=2, kmax=8)
    base.update(ov)
    w = get_config("tiny", **base)
    Q, K, V = make_qkv(w)
    res = run_library(w, Q, K, V)
    assert res["status"] == 0
    _assert_ok(oracle_check(w, Q, K, V, res))
    nb = w.nb
    k = np.diff(res["row_ptr"])
    assert np.all(k >= min(w.kmin, nb)) and np.all(k <= min(w.kmax, nb))
