"""The FMA-pipe base-2 exponential used for part of the softmax (tc::ex2_fma).

Its coefficients live in the CUDA header; this CPU test reads them from there
and replays the same float32 steps (round-to-integer split, degree-3
polynomial, exponent add) with numpy, checking the relative error against
exp2 over the exponent range the softmax uses.  The bound (1e-4) is far below
the 2^-9 relative rounding of the bf16 probabilities the values feed.
"""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "block_sparse_attention_33_b200", "csrc", "tc.cuh")


def coeffs():
    src = open(HDR).read()
    return [np.float32(float(re.search(rf"kExp2C{k} = ([0-9.eE+-]+)f", src).group(1)))
            for k in range(4)]


def fma32(a, b, c):
    return (a.astype(np.float64) * b + c).astype(np.float32)


def ex2_fma(x):
    c0, c1, c2, c3 = coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-125))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - n).astype(np.float32)
    q = fma32(fma32(fma32(np.full_like(f, c3), f, c2), f, c1), f, c0)
    ni = t.view(np.int32) - np.int32(0x4B400000)
    return (q.view(np.int32) + (ni << 23)).view(np.float32)


def test_ex2_fma_relative_error_bound():
    x = np.concatenate([np.linspace(-125, 8, 2_000_001, dtype=np.float32),
                        np.array([0, -0.5, 0.5, 1, -1, 7.99, -124.5], np.float32)])
    got = ex2_fma(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1e-4, rel.max()


def test_ex2_fma_clamps_far_below_range():
    x = np.array([-200.0, -1e30, -np.inf], np.float32)
    got = ex2_fma(x)
    assert np.all(np.isfinite(got)) and np.all(got < 1e-37) and np.all(got > 0)


def test_coefficients_are_a_fit_of_exp2():
    # sanity: at f = 0 the polynomial is ~1, its slope ~ln 2
    c0, c1, _, _ = coeffs()
    assert abs(c0 - 1) < 1e-4 and abs(c1 - np.log(2)) < 2e-3


def test_paired_exponent_add_matches_scalar():
    """The paired form adds bits(t) << 23 instead of n << 23; the two agree
    modulo 2^32 because the low nine bits of bits(1.5 * 2^23) are zero."""
    x = np.linspace(-125, 8, 100_001, dtype=np.float32)
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n_shift = ((t.view(np.int32) - np.int32(0x4B400000)).astype(np.int64) << 23) & 0xFFFFFFFF
    t_shift = (t.view(np.uint32).astype(np.int64) << 23) & 0xFFFFFFFF
    assert np.array_equal(n_shift, t_shift)


def _remez_relative(deg, iters=30):
    """Minimax fit of 2^f on [-1/2, 1/2] in relative error by the Remez
    exchange: solve p(x_i) + (-1)^i E 2^(x_i) = 2^(x_i) on deg + 2 reference
    points, move the points to the extrema of the new error curve, repeat.
    Returns (coefficients low to high, max relative error on a fine grid)."""
    n = deg + 2
    x = 0.5 * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))   # Chebyshev extrema
    t = np.linspace(-0.5, 0.5, 200_001)
    err = None
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * np.exp2(x[i])
        c = np.linalg.solve(A, np.exp2(x))[:deg + 1]
        err = (np.polyval(c[::-1], t) - np.exp2(t)) / np.exp2(t)
        segs = np.split(np.arange(len(t)), np.nonzero(np.diff(np.sign(err)) != 0)[0] + 1)
        ext = [s[np.argmax(np.abs(err[s]))] for s in segs]
        if len(ext) != n:
            break
        x = t[ext]
    return c, float(np.max(np.abs(err)))


def test_coefficients_are_the_degree_3_relative_minimax_fit():
    """The header's constants are the float32 roundings of the degree-3
    relative-error minimax polynomial of 2^f on [-1/2, 1/2], re-derived here
    by the Remez exchange; its error equioscillates at about 7.5e-5."""
    c, emax = _remez_relative(3)
    assert np.array_equal(np.float32(c), np.array(coeffs(), np.float32)), (np.float32(c), coeffs())
    assert 7.0e-5 < emax < 8.0e-5
    # a degree lower is far worse, so degree 3 is the smallest that fits the bf16 budget
    _, e2 = _remez_relative(2)
    assert e2 > 1e-3
