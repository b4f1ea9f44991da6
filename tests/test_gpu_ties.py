"""Exact ties in the routing through the C ABI.  Zero queries and keys make
every proxy logit ln b, so with 16 full blocks every p is exactly 1/16 in
fp32 and fp64 alike and every prefix mass is exact; the tie rule (the lower
block first) then fixes the kept set uniquely, for Top-p, PAMA and the
threshold selection, on both attention kernels."""
import numpy as np
import pytest

from tests.harness import MAX_ABS, REL_L2, oracle_check, run_library
from workloads import get_config, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu(gpu_required):
    import block_sparse_attention_33_b200 as sp
    sp.lib()


def _assert_ok(fig):
    assert fig["bad"] == 0, fig
    assert fig["max_abs"] < MAX_ABS and fig["rel_l2"] < REL_L2, fig


# Exact ties: zero queries and keys make every proxy logit ln b, so with 16
# full blocks every p is exactly 1/16 in fp32 and fp64 alike and every prefix
# mass is exact.  The tie rule (lower block first) then fixes the kept set
# uniquely; the oracle comparison alone would accept any choice among the
# tied blocks, since it marks them marginal.
TIES = [
    # (description, config overrides, routing flags, tau or theta, kmin, expected kept blocks)
    ("top-p 0.3 keeps 5 (warp MMA)", dict(), 0, 0.3, 1, list(range(5))),
    ("top-p 0.3 keeps 5 (tcgen05)", dict(grid=(2, 8, 128), d=128, b=128), 0, 0.3, 1, list(range(5))),
    ("top-p 0.5 keeps 8, PAMA", dict(), 1, 0.5, 1, list(range(8))),
    ("theta 1/16 keeps all", dict(), 16, 0.0625, 1, list(range(16))),
    ("theta above 1/16, kmin 3", dict(), 16, 0.07, 3, [0, 1, 2]),
]


@pytest.mark.parametrize("desc,ov,flags,tau,kmin,want", TIES, ids=[t[0] for t in TIES])
def test_exact_ties_break_to_the_lower_block(desc, ov, flags, tau, kmin, want):
    base = dict(H=2, kmin=kmin, kmax=16, tau=tau)
    base.update(ov)
    w = get_config("tiny", **base)
    assert w.nb == 16 and w.N % w.b == 0
    _, _, V = make_qkv(w)
    Z = np.zeros(V.shape, np.uint16)                      # bf16 +0.0
    res = run_library(w, Z, Z, V, routing=flags)
    assert res["status"] == 0
    k = np.diff(res["row_ptr"])
    assert np.all(k == len(want)), k
    for r in range(w.B * w.H * w.nb):
        assert res["col_idx"][res["row_ptr"][r]:res["row_ptr"][r + 1]].tolist() == want
    sel = "threshold" if flags & 16 else "top_p"
    _assert_ok(oracle_check(w, Z, Z, V, res, routing="pama" if flags & 1 else "centroid",
                            selection=sel))
