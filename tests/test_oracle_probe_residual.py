"""Pins for the probe-fitted residual correction of the oracle (SparsePR page,
section 2B): a hand-worked one-dimensional case, scikit-learn's ridge
regression with an intercept, exact recovery of an affine low-rank residual,
the two limits of the penalty, a known residual subspace, and library
softmax attention for the exact probe rows.  A transposed B, a penalised
bias, a projector built from left instead of right singular vectors, or
probe rows left uncorrected each fail one of them.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch
from sklearn.linear_model import Ridge

from oracle import probe_residual as P
from oracle import spattn_ref as R
from workloads import get_config, make_qkv, probe_rows


def test_one_dimensional_fit_by_hand():
    # x = 1, 2, 4 and residuals 3, 1, 2: with the bias unpenalised the slope
    # is Sxy / (Sxx + lam) over centred data and the bias ybar - slope * xbar.
    x = [Fraction(1), Fraction(2), Fraction(4)]
    y = [Fraction(3), Fraction(1), Fraction(2)]
    lam = Fraction(1, 2)
    xb, yb = sum(x) / 3, sum(y) / 3
    sxy = sum((a - xb) * (c - yb) for a, c in zip(x, y))
    sxx = sum((a - xb) ** 2 for a in x)
    slope = sxy / (sxx + lam)
    bias = yb - slope * xb
    X = np.array([[float(a)] for a in x])
    Y = np.array([[float(c)] for c in y])
    b_, B_ = P.fit_affine_residual(X, Y, float(lam))
    assert b_[0] == pytest.approx(float(bias), abs=1e-14)
    assert B_[0, 0] == pytest.approx(float(slope), abs=1e-14)
    # one output dimension, non-zero residual: the projector is 1, so every
    # unprobed row gets bias + slope * x and probe rows their exact value
    O = np.array([[1.0], [2.0], [4.0], [3.0], [-1.0]])
    out = P.correct(O, O[[0, 1, 2]] + Y, np.array([0, 1, 2]), float(lam), 1)
    for i, xi in ((3, 3.0), (4, -1.0)):
        assert out[i, 0] == pytest.approx(xi + float(bias) + float(slope) * xi, abs=1e-13)
    np.testing.assert_allclose(out[:3], O[:3] + Y, rtol=0, atol=1e-15)


@pytest.mark.parametrize("lam", [1e-3, 0.7, 25.0])
def test_fit_matches_sklearn_ridge_with_intercept(lam):
    rng = np.random.default_rng(11)
    X = rng.standard_normal((40, 6))
    Y = rng.standard_normal((40, 5)) + X @ rng.standard_normal((6, 5))
    b_, B_ = P.fit_affine_residual(X, Y, lam)
    ref = Ridge(alpha=lam, fit_intercept=True, solver="svd").fit(X, Y)
    np.testing.assert_allclose(B_, ref.coef_.T, rtol=0, atol=1e-10)
    np.testing.assert_allclose(b_, ref.intercept_, rtol=0, atol=1e-10)


def test_full_rank_projector_gives_the_plain_ridge_prediction():
    rng = np.random.default_rng(12)
    N, d, m = 80, 6, 30
    O = rng.standard_normal((N, d))
    probes = np.sort(rng.choice(N, m, replace=False))
    exact = O[probes] + rng.standard_normal((m, d))
    out = P.correct(O, exact, probes, 0.3, d)
    ref = Ridge(alpha=0.3, fit_intercept=True, solver="svd").fit(O[probes], exact - O[probes])
    rest = np.setdiff1d(np.arange(N), probes)
    np.testing.assert_allclose(out[rest], O[rest] + ref.predict(O[rest]), rtol=0, atol=1e-10)


def test_affine_low_rank_residual_is_recovered_exactly():
    rng = np.random.default_rng(13)
    N, d, m, r0 = 200, 16, 40, 3
    U = np.linalg.qr(rng.standard_normal((d, r0)))[0]          # residual subspace
    b0 = U @ rng.standard_normal(r0)
    B0 = rng.standard_normal((d, r0)) @ U.T
    O = rng.standard_normal((N, d))
    truth = O + b0[None, :] + O @ B0
    probes = probe_rows(N, 5, 0)[:m]
    out = P.correct(O, truth[probes], probes, 1e-12, r0)
    np.testing.assert_allclose(out, truth, rtol=0, atol=1e-8)


def test_correction_stays_in_the_residual_subspace():
    rng = np.random.default_rng(14)
    N, d, m, r0 = 120, 10, 30, 2
    U = np.linalg.qr(rng.standard_normal((d, r0)))[0]
    O = rng.standard_normal((N, d))
    probes = np.arange(0, N, N // m)[:m]
    resid = rng.standard_normal((m, r0)) @ U.T                  # rows in span(U), not affine in O
    out = P.correct(O, O[probes] + resid, probes, 0.5, r0)
    C = out - O
    rest = np.setdiff1d(np.arange(N), probes)
    off = C[rest] - C[rest] @ U @ U.T
    assert np.abs(off).max() < 1e-12
    assert np.abs(C[rest]).max() > 1e-3                         # and it is not trivially zero


def test_rank_zero_and_infinite_penalty_limits():
    rng = np.random.default_rng(15)
    N, d, m = 60, 8, 20
    O = rng.standard_normal((N, d))
    probes = np.arange(0, N, 3)[:m]
    exact = O[probes] + rng.standard_normal((m, d)) + 2.0
    rest = np.setdiff1d(np.arange(N), probes)
    # r = 0: no correction off the probes, exact values on them
    out = P.correct(O, exact, probes, 0.1, 0)
    np.testing.assert_array_equal(out[rest], O[rest])
    np.testing.assert_array_equal(out[probes], exact)
    # lam -> infinity: B -> 0, the bias -> the mean probe residual, so every
    # unprobed row moves by the same vector, the projected mean residual
    Rm = exact - O[probes]
    _, _, Vt = torch.linalg.svd(torch.from_numpy(Rm), full_matrices=False)
    V = Vt[:3].T.numpy()
    out = P.correct(O, exact, probes, 1e14, 3)
    shift = Rm.mean(axis=0) @ V @ V.T
    np.testing.assert_allclose(out[rest] - O[rest], np.broadcast_to(shift, (len(rest), d)),
                               rtol=0, atol=1e-9)


def test_dense_rows_match_library_attention():
    rng = np.random.default_rng(16)
    N, d = 150, 32
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    rows = np.array([0, 7, 64, 149])
    t = lambda x: torch.from_numpy(x)[None, None]
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v))[0, 0].numpy()
    np.testing.assert_allclose(P.dense_rows(q, k, v, rows), ref[rows], rtol=0, atol=1e-13)


def test_forward_probe_keeps_probes_exact_and_shrinks_the_error():
    """On the tiny video-like workload routed to two key blocks per query
    block, with two probe rows per output dimension and a strong penalty,
    the corrected output is exact on the probe rows and closer to dense
    attention elsewhere than the routed output it starts from."""
    w = get_config("tiny")
    Q, K, V = make_qkv(w)
    B, H, N, d = Q.shape
    probes = np.stack([np.stack([probe_rows(N, w.b, (5, bi, hi), 16) for hi in range(H)])
                       for bi in range(B)])
    res = P.forward_probe(Q, K, V, w.b, w.tau, 1, 2, 1, probes, 100.0, d)
    for hi in range(H):
        q, k, v = (R.decode_bf16(X[0, hi]) for X in (Q, K, V))
        dense = P.dense_rows(q, k, v, np.arange(N))
        rows = probes[0, hi]
        np.testing.assert_array_equal(res["O"][0, hi][rows], dense[rows])
        rest = np.setdiff1d(np.arange(N), rows)
        e_sparse = np.linalg.norm(res["O_sparse"][0, hi][rest] - dense[rest])
        e_corr = np.linalg.norm(res["O"][0, hi][rest] - dense[rest])
        assert e_corr < 0.99 * e_sparse


def test_row_subset_evaluation_equals_the_full_evaluation():
    """forward_probe(rows=...) evaluates the routed output only at the probes
    and the requested rows; the corrected rows (probe rows among them) equal
    those of the full evaluation, and the routing is the same."""
    w = get_config("tiny", kmax=2)
    Q, K, V = make_qkv(w)
    B, H, N, d = Q.shape
    probes = np.stack([np.stack([probe_rows(N, w.b, (5, bi, hi), 4) for hi in range(H)])
                       for bi in range(B)])
    full = P.forward_probe(Q, K, V, w.b, w.tau, w.kmin, w.kmax, w.residual, probes, 100.0, 8)
    rng = np.random.default_rng(2)
    rows = {(0, hi): np.sort(np.concatenate([rng.choice(N, 30, replace=False), probes[0, hi][:3]]))
            for hi in range(H)}
    sub = P.forward_probe(Q, K, V, w.b, w.tau, w.kmin, w.kmax, w.residual, probes, 100.0, 8,
                          rows=rows)
    for hi in range(H):
        np.testing.assert_array_equal(sub["O"][(0, hi)], full["O"][0, hi][rows[(0, hi)]])
        np.testing.assert_array_equal(sub["O_sparse"][(0, hi)],
                                      full["O_sparse"][0, hi][rows[(0, hi)]])
        for a, b in zip(sub["route"][(0, hi)]["kept"], full["route"][(0, hi)]["kept"]):
            np.testing.assert_array_equal(a, b)
