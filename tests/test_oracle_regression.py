"""The oracle against its own recorded output on the tiny layer
(tests/golden/oracle_regression_tiny.txt, written by
tests/golden/make_oracle_regression.py from the oracle alone).  A regression
guard, not a correctness pin: the pins elsewhere tie the oracle to the pages;
this test makes any later change to its arithmetic visible and deliberate.
Kept sets must match exactly; outputs to 1e-12 relative (BLAS threading may
reorder sums)."""
import os

import numpy as np

from oracle import probe_residual as P
from oracle import spattn_ref as R
from workloads import get_config, make_qkv, probe_rows

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "oracle_regression_tiny.txt")


def _records(tag):
    for line in open(GOLDEN):
        if line.startswith(tag + " "):
            _, bi, hi, idx, *vals = line.split()
            yield int(bi), int(hi), int(idx), vals


def test_oracle_matches_its_recorded_output():
    w = get_config("tiny")
    Q, K, V = make_qkv(w)
    res = R.forward(Q, K, V, w.b, w.tau, w.kmin, w.kmax, w.residual)
    kept = list(_records("kept"))
    for bi, hi, i, vals in kept:
        assert res["route"][(bi, hi)]["kept"][i].tolist() == [int(v) for v in vals], (bi, hi, i)
    outs = list(_records("out"))
    for bi, hi, n, vals in outs:
        np.testing.assert_allclose(res["O"][bi, hi, n], np.array(vals, float), rtol=1e-12, atol=1e-14)
    assert len(kept) == w.B * w.H * w.nb and len(outs) == w.B * w.H * 8


def test_threshold_and_probe_correction_match_their_recorded_output():
    w = get_config("tiny")
    Q, K, V = make_qkv(w)
    thr = R.forward(Q, K, V, w.b, 0.05, w.kmin, w.kmax, w.residual, want_output=False,
                    selection="threshold")
    kept = list(_records("kept_threshold"))
    for bi, hi, i, vals in kept:
        assert thr["route"][(bi, hi)]["kept"][i].tolist() == [int(v) for v in vals], (bi, hi, i)
    probes = np.stack([np.stack([probe_rows(w.N, w.b, (5, bi, hi), 16) for hi in range(w.H)])
                       for bi in range(w.B)])
    pc = P.forward_probe(Q, K, V, w.b, w.tau, 1, 2, 1, probes, 100.0, 16)
    outs = list(_records("out_probe"))
    for bi, hi, n, vals in outs:
        np.testing.assert_allclose(pc["O"][bi, hi, n], np.array(vals, float), rtol=1e-10, atol=1e-12)
    assert len(kept) == w.B * w.H * w.nb and len(outs) == w.B * w.H * 8
