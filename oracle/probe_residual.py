"""Probe-fitted residual reconstruction, plain fp64 reference (test
infrastructure only; the product path never imports it).

SparsePR page, section 2B: a few query rows (probes) are evaluated exactly;
their residual R = O_dense - O_sparse is modelled as an affine function of
the sparse output, R ~ b + x B, fitted per attention call by ridge
regression; the fitted correction is restricted to the subspace spanned by
the leading right singular vectors of the probe residuals and added to the
sparse output of every other row.  Probe rows keep their exact output.

Readings of points the page leaves open:

* the fit is per (batch, head): one attention call per head;
* probes are an input (random draws of the method, made by the seeded
  generator workloads.probe_rows: the same number of tokens from every
  query block at seeded offsets, i.e. stratified across query groups, the
  page's groups being the blocks here); the probe count is a parameter,
  since the page gives none;
* the ridge penalty lam applies to B only, not to the bias b (the usual
  ridge-with-intercept);
* the subspace is that of the r leading right singular vectors of R (the
  probe residual matrix itself, without centring); r = 0 disables the
  correction.
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np

from . import spattn_ref


def fit_affine_residual(X: np.ndarray, R: np.ndarray, lam: float):
    """Ridge fit of R ~ 1 b + X B with the penalty lam ||B||^2 (the bias is
    not penalised): returns (b [d_out], B [d_in, d_out]).  Solved from the
    normal equations of the augmented design [1, X]."""
    m, d_in = X.shape
    A = np.concatenate([np.ones((m, 1)), X], axis=1)
    D = np.eye(d_in + 1) * lam
    D[0, 0] = 0.0
    W = np.linalg.solve(A.T @ A + D, A.T @ R)
    return W[0], W[1:]


def residual_subspace(R: np.ndarray, r: int) -> np.ndarray:
    """Projector onto the span of the r leading right singular vectors of
    the probe residuals R [m, d]: [d, d]."""
    d = R.shape[1]
    if r <= 0:
        return np.zeros((d, d))
    _, _, Vt = np.linalg.svd(R, full_matrices=False)
    Vr = Vt[:r].T
    return Vr @ Vr.T


def fit_correction(X: np.ndarray, O_dense_probe: np.ndarray, lam: float, r: int):
    """The fitted correction of one head from its probe rows: X [m, d] the
    sparse output at the probes, O_dense_probe [m, d] their exact output.
    Returns (bias, B, P): a row x is corrected to x + (bias + x B) P."""
    R = O_dense_probe - X
    bias, B = fit_affine_residual(X, R, lam)
    return bias, B, residual_subspace(R, r)


def correct(O_sparse: np.ndarray, O_dense_probe: np.ndarray, probes: np.ndarray, lam: float,
            r: int) -> np.ndarray:
    """The corrected output of one head: O_sparse [N, d] plus the projected
    affine correction on every row; probe rows take their exact output."""
    bias, B, P = fit_correction(O_sparse[probes], O_dense_probe, lam, r)
    C = (bias[None, :] + O_sparse @ B) @ P
    out = O_sparse + C
    out[probes] = O_dense_probe
    return out


def dense_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, rows: np.ndarray) -> np.ndarray:
    """Exact softmax attention of the query rows `rows` over every key
    (scale 1/sqrt(d)), fp64: [len(rows), d]."""
    z = q[rows] @ k.T / math.sqrt(q.shape[1])
    w = np.exp(z - z.max(axis=1, keepdims=True))
    return (w @ v) / w.sum(axis=1, keepdims=True)


def forward_probe(Q, K, V, b: int, tau: float, kmin: int, kmax: int, residual: int,
                  probes: np.ndarray, lam: float, r: int, perm: Optional[np.ndarray] = None,
                  routing: str = "centroid", rows: Optional[dict] = None):
    """The routed path followed by the probe-fitted correction, per head.

    probes: [B, H, M] token indices in the ORIGINAL order (an input, so that
    any implementation corrects with the same probes).
    rows:   optional {(b, h): token indices in the ORIGINAL order}: only those
            corrected rows are computed.  The routed output is then evaluated
            at the probes and at those rows alone (the fit needs the sparse
            output at the probes only), which gives the same rows as the full
            evaluation.
    Returns the routed result of spattn_ref.forward with O replaced by the
    corrected output and O_sparse holding the uncorrected one (arrays
    [B, H, N, d], or with `rows` dicts {(b, h): [len(rows), d]})."""
    if rows is not None:
        return _forward_probe_rows(Q, K, V, b, tau, kmin, kmax, residual, probes, lam, r, perm,
                                   routing, rows)
    res = spattn_ref.forward(Q, K, V, b, tau, kmin, kmax, residual, perm=perm, routing=routing)
    O_sparse = res["O"]
    O = np.empty_like(O_sparse)
    B, H = Q.shape[:2]
    for bi in range(B):
        for hi in range(H):
            q = spattn_ref.decode_bf16(Q[bi, hi])
            k = spattn_ref.decode_bf16(K[bi, hi])
            v = spattn_ref.decode_bf16(V[bi, hi])
            rows = np.asarray(probes[bi, hi], dtype=np.int64)
            O[bi, hi] = correct(O_sparse[bi, hi], dense_rows(q, k, v, rows), rows, lam, r)
    res["O_sparse"] = O_sparse
    res["O"] = O
    return res


def _forward_probe_rows(Q, K, V, b, tau, kmin, kmax, residual, probes, lam, r, perm, routing,
                        rows):
    """forward_probe restricted to the rows of `rows` (see there)."""
    B, H = Q.shape[:2]
    need = {(bi, hi): np.union1d(np.asarray(probes[bi, hi], dtype=np.int64),
                                 np.asarray(rows[(bi, hi)], dtype=np.int64))
            for bi in range(B) for hi in range(H)}
    res = spattn_ref.forward(Q, K, V, b, tau, kmin, kmax, residual, perm=perm, rows=need,
                             routing=routing)
    O, O_sparse = {}, {}
    for bi in range(B):
        for hi in range(H):
            key = (bi, hi)
            q = spattn_ref.decode_bf16(Q[bi, hi])
            k = spattn_ref.decode_bf16(K[bi, hi])
            v = spattn_ref.decode_bf16(V[bi, hi])
            pr = np.asarray(probes[bi, hi], dtype=np.int64)
            want = np.asarray(rows[key], dtype=np.int64)
            sub = res["O"][key]                          # sparse output at need[key]
            x_want = sub[np.searchsorted(need[key], want)]
            dense = dense_rows(q, k, v, pr)
            bias, Bm, P = fit_correction(sub[np.searchsorted(need[key], pr)], dense, lam, r)
            out = x_want + (bias[None, :] + x_want @ Bm) @ P
            for e, t in enumerate(want):
                hit = np.nonzero(pr == t)[0]
                if len(hit):
                    out[e] = dense[hit[0]]               # a probe row takes its exact output
            O[key], O_sparse[key] = out, x_want
    res["O_sparse"] = O_sparse
    res["O"] = O
    return res
