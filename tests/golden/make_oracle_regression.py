"""Writes tests/golden/oracle_regression_tiny.txt from the oracle alone.

A regression fixture, not a correctness pin: it records what the fp64
oracle computes today on the tiny layer (B1 H2 d64, 4x16x16 grid, b = 64,
tau = 0.9, kmin 1, kmax 16, residual on): every head's kept blocks per query
block, and eight output rows per head at full precision; the kept blocks of
the threshold selection at theta = 0.05; and eight rows per head of the
probe-fitted correction (kmax 2, 16 probes per block, lam = 100, r = 16).  A later change to
the oracle's arithmetic shows up as a diff of this file; such a change names
the passage of the pages, or the reading of it, that justifies it.

    python tests/golden/make_oracle_regression.py
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import probe_residual as P                  # noqa: E402
from oracle import spattn_ref as R                     # noqa: E402
from workloads import get_config, make_qkv, probe_rows  # noqa: E402

ROWS = (0, 1, 63, 64, 511, 512, 960, 1023)
OUT = os.path.join(HERE, "oracle_regression_tiny.txt")


def main():
    w = get_config("tiny")
    Q, K, V = make_qkv(w)
    res = R.forward(Q, K, V, w.b, w.tau, w.kmin, w.kmax, w.residual)
    lines = ["# oracle regression fixture, tiny layer (written by make_oracle_regression.py)"]
    for (bi, hi), r in sorted(res["route"].items()):
        for i, kept in enumerate(r["kept"]):
            lines.append(f"kept {bi} {hi} {i} " + " ".join(str(int(j)) for j in kept))
    for bi in range(w.B):
        for hi in range(w.H):
            for n in ROWS:
                vals = " ".join(f"{x:.17g}" for x in res["O"][bi, hi, n])
                lines.append(f"out {bi} {hi} {n} {vals}")
    thr = R.forward(Q, K, V, w.b, 0.05, w.kmin, w.kmax, w.residual, want_output=False,
                    selection="threshold")
    for (bi, hi), r in sorted(thr["route"].items()):
        for i, kept in enumerate(r["kept"]):
            lines.append(f"kept_threshold {bi} {hi} {i} " + " ".join(str(int(j)) for j in kept))
    probes = np.stack([np.stack([probe_rows(w.N, w.b, (5, bi, hi), 16) for hi in range(w.H)])
                       for bi in range(w.B)])
    pc = P.forward_probe(Q, K, V, w.b, w.tau, 1, 2, 1, probes, 100.0, 16)
    for bi in range(w.B):
        for hi in range(w.H):
            for n in ROWS:
                vals = " ".join(f"{x:.17g}" for x in pc["O"][bi, hi, n])
                lines.append(f"out_probe {bi} {hi} {n} {vals}")
    with open(OUT, "w") as f:
        f.write("\n".join(lines) + "\n")


if __name__ == "__main__":
    main()
