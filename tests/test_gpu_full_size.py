"""Full-size workloads: routing checked on every query block, outputs on samples.

At these sizes the fp64 oracle cannot evaluate every output row, so it
evaluates a stated sample per head: tokens of the partial last query block,
of the query block with the largest budget, and of two random query blocks
(first, last and one random row of each).  Routing is compared on all rows.
"""
import numpy as np
import pytest

from tests.harness import oracle_check, run_library
from workloads import get_config, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu(gpu_required):
    import block_sparse_attention_33_b200 as sp
    sp.lib()


def sample_rows(w, res, perm, seed=0):
    rng = np.random.default_rng(seed)
    nb, b = res["nb"], w.b
    rows = {}
    for bi in range(w.B):
        for hi in range(w.H):
            base = (bi * w.H + hi) * nb
            k = np.diff(res["row_ptr"][base: base + nb + 1])
            blocks = {nb - 1, int(np.argmax(k))} | set(rng.integers(0, nb, 2).tolist())
            picked = []
            for i in sorted(blocks):
                n_i = min(b, w.N - i * b)
                for r in {0, n_i - 1, int(rng.integers(0, n_i))}:
                    picked.append(i * b + r)          # blocked (permuted) order
            picked = np.array(sorted(picked))
            rows[(bi, hi)] = picked if perm is None else np.asarray(perm)[picked]
    return rows


CASES = [
    ("wan", dict(tau=0.8)), ("wan", dict(tau=0.9)), ("wan", dict(tau=0.95)),
    ("hunyuan", dict(tau=0.8)), ("hunyuan", dict(tau=0.95)),
    ("stress", dict(residual=1)), ("stress", dict(residual=0)),
]


@pytest.mark.parametrize("name,ov", CASES, ids=[f"{n}-{ov}" for n, ov in CASES])
def test_full_size(name, ov):
    w = get_config(name, **ov)
    Q, K, V = make_qkv(w)
    perm = None
    if w.hilbert:
        import block_sparse_attention_33_b200 as sp
        perm = sp.spattn_hilbert_perm(*w.grid)
    res = run_library(w, Q, K, V, perm=perm)
    assert res["status"] == 0
    rows = sample_rows(w, res, perm)
    fig = oracle_check(w, Q, K, V, res, perm=perm, rows=rows)
    print(f"\n{name} {ov}: kept fraction {fig['kept_fraction']:.4f}, marginal flips "
          f"{fig['marginal']} in {fig['rows_diff']} rows, max-abs {fig['max_abs']:.2e}, "
          f"rel-L2 {fig['rel_l2']:.2e}")
    assert fig["bad"] == 0, fig
    assert fig["max_abs"] < 2e-2 and fig["rel_l2"] < 4e-3, fig


def test_largest_supported_block_count():
    """nb = 2048 (the supported maximum): 262144 tokens of one head in
    128-token blocks, through the tcgen05 path, sixteen centroid tiles per
    item in residual mode; sampled rows against the oracle."""
    w = get_config("tiny", grid=(1, 512, 512), d=128, b=128, H=1, kmax=16, tau=0.9)
    assert w.nb == 2048
    Q, K, V = make_qkv(w)
    res = run_library(w, Q, K, V)
    assert res["status"] == 0
    rows = sample_rows(w, res, None)
    fig = oracle_check(w, Q, K, V, res, rows=rows)
    assert fig["bad"] == 0, fig
    assert fig["max_abs"] < 2e-2 and fig["rel_l2"] < 4e-3, fig
