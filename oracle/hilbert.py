"""3D Hilbert token order (test infrastructure only).

The DFSAttn abstract (thelatestinai page) reorders tokens along a Hilbert
curve before blocking, so that each block of b consecutive tokens is a
compact 3D patch of the (t, h, w) latent grid.  The pages do not say which
Hilbert curve; the reading taken here is J. Skilling's construction
("Programming the Hilbert curve", AIP Conf. Proc. 707, 2004):

* axes in the order X0 = t, X1 = h, X2 = w, each coordinate written with
  ``bits`` bits, where 2**bits is the smallest power of two that covers the
  largest grid side (a 21x30x52 grid lives in the 64^3 cube);
* the transform walks the bit levels from the top, at each level either
  inverting the lower bits of X0 or exchanging them with Xi, then
  Gray-encodes across the axes;
* the Hilbert index reads the transformed words level by level from the most
  significant bit, X0 first.

Tokens are then stably sorted by that index; perm[new] = old.

This is a vectorised restatement over all cells at once, written from the
published description; the pins in the tests check it is a Hilbert curve
(bijective, every step a unit move, order 1 = binary-reflected Gray code).
"""
from __future__ import annotations

import numpy as np


def hilbert_index(coords: np.ndarray, bits: int) -> np.ndarray:
    """coords: [M, n] non-negative ints < 2**bits -> Hilbert index [M] (int64)."""
    X = np.array(coords, dtype=np.int64, copy=True)
    n = X.shape[1]
    top = 1 << (bits - 1)
    # level walk: invert or exchange the bits below the current level
    Q = top
    while Q > 1:
        P = Q - 1
        for i in range(n):
            hit = (X[:, i] & Q) != 0
            X[hit, 0] ^= P
            t = (X[~hit, 0] ^ X[~hit, i]) & P
            X[~hit, 0] ^= t
            X[~hit, i] ^= t
        Q >>= 1
    # Gray encode across the axes
    for i in range(1, n):
        X[:, i] ^= X[:, i - 1]
    t = np.zeros(X.shape[0], dtype=np.int64)
    Q = top
    while Q > 1:
        t ^= np.where((X[:, n - 1] & Q) != 0, Q - 1, 0)
        Q >>= 1
    X ^= t[:, None]
    # interleave: level by level from the top, axis 0 most significant
    h = np.zeros(X.shape[0], dtype=np.int64)
    for level in range(bits - 1, -1, -1):
        for i in range(n):
            h = (h << 1) | ((X[:, i] >> level) & 1)
    return h


def hilbert_perm(grid) -> np.ndarray:
    """perm[new] = old for a T x Hs x W grid in row-major token order."""
    T, Hs, W = grid
    side = max(T, Hs, W)
    bits = max(1, int(np.ceil(np.log2(side))))
    t, h, w = np.meshgrid(np.arange(T), np.arange(Hs), np.arange(W), indexing="ij")
    coords = np.stack([t.ravel(), h.ravel(), w.ravel()], axis=1)
    key = hilbert_index(coords, bits)
    return np.argsort(key, kind="stable").astype(np.int64)
