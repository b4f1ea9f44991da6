"""The oracle against its own recorded output on the tiny layer
(tests/golden/oracle_regression_tiny.txt, written by
tests/golden/make_oracle_regression.py from the oracle alone).  A regression
guard, not a correctness pin: the pins elsewhere tie the oracle to the pages;
this test makes any later change to its arithmetic visible and deliberate.
Kept sets must match exactly; outputs to 1e-12 relative (BLAS threading may
reorder sums)."""
import os

import numpy as np

from oracle import spattn_ref as R
from workloads import get_config, make_qkv

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "oracle_regression_tiny.txt")


def test_oracle_matches_its_recorded_output():
    w = get_config("tiny")
    Q, K, V = make_qkv(w)
    res = R.forward(Q, K, V, w.b, w.tau, w.kmin, w.kmax, w.residual)
    n_kept = n_out = 0
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        tag, bi, hi, idx, *vals = line.split()
        bi, hi, idx = int(bi), int(hi), int(idx)
        if tag == "kept":
            assert res["route"][(bi, hi)]["kept"][idx].tolist() == [int(v) for v in vals], (bi, hi, idx)
            n_kept += 1
        else:
            want = np.array([float(v) for v in vals])
            np.testing.assert_allclose(res["O"][bi, hi, idx], want, rtol=1e-12, atol=1e-14)
            n_out += 1
    assert n_kept == w.B * w.H * w.nb and n_out == w.B * w.H * 8
