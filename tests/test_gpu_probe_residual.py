"""Probe-fitted residual correction (SparsePR page, section 2B) through the C
ABI against the oracle: the library's routed output is corrected on the GPU
and, from the same routed output, by oracle.probe_residual.correct with the
oracle's own exact probe rows; the two must agree within the output bounds,
and the probe rows must hold their exact output."""
import numpy as np
import pytest

from oracle import probe_residual as P
from oracle import spattn_ref as R
from tests.harness import MAX_ABS, REL_L2, compare_outputs, from_dev, to_dev
from workloads import get_config, make_qkv, probe_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu(gpu_required):
    import block_sparse_attention_33_b200 as sp
    sp.lib()


def _run(w, per_block, lam, r, bad_probe=False):
    import torch
    import block_sparse_attention_33_b200 as sp
    Q, K, V = make_qkv(w)
    probes = np.stack([np.stack([probe_rows(w.N, w.b, (5, bi, hi), per_block)
                                 for hi in range(w.H)]) for bi in range(w.B)]).astype(np.int32)
    if bad_probe:
        probes[0, 0, 0] = w.N + 3
    plan = sp.Plan(w.B, w.H, w.N, w.d, w.b, w.tau, w.kmin, w.kmax, w.residual)
    try:
        q, k, v = to_dev(Q), to_dev(K), to_dev(V)
        o = torch.zeros_like(q)
        plan.forward(q, k, v, o)
        assert plan.check() == sp.OK
        o_sparse = from_dev(o)
        plan.probe_correct(q, k, v, o, torch.from_numpy(probes).cuda(), lam, r)
        status = plan.check()
        return Q, K, V, probes, o_sparse, from_dev(o), status
    finally:
        plan.close()


CASES = [
    ("tiny d=64, r=16", "tiny", dict(kmax=2), 16, 100.0, 16),
    ("medium 2 heads, r=8", "medium", dict(H=2, tau=0.8), 4, 100.0, 8),
    ("medium 2 heads, r=d", "medium", dict(H=2, tau=0.8), 4, 10.0, 128),
    ("medium 2 heads, r=0", "medium", dict(H=2, tau=0.8), 2, 100.0, 0),
    ("wan 2 heads (512 key tiles), r=8", "wan", dict(H=2), 1, 100.0, 8),
]


@pytest.mark.parametrize("desc,name,ov,per_block,lam,r", CASES, ids=[c[0] for c in CASES])
def test_probe_correction_against_oracle(desc, name, ov, per_block, lam, r):
    import block_sparse_attention_33_b200 as sp
    w = get_config(name, **ov)
    Q, K, V, probes, o_sparse, o_corr, status = _run(w, per_block, lam, r)
    assert status == sp.OK
    for bi in range(w.B):
        for hi in range(w.H):
            q, k, v = (R.decode_bf16(X[bi, hi]) for X in (Q, K, V))
            rows = probes[bi, hi].astype(np.int64)
            dense = P.dense_rows(q, k, v, rows)
            want = P.correct(o_sparse[bi, hi], dense, rows, lam, r)
            max_abs, rel = compare_outputs(o_corr[bi, hi], want)
            assert max_abs < MAX_ABS and rel < REL_L2, (bi, hi, max_abs, rel)
            # probe rows: the exact output (fp32 on the device), one bf16 rounding (at most
            # 2^-8 relative)
            assert (np.abs(o_corr[bi, hi][rows] - dense).max()
                    <= 2.0 ** -8 * np.abs(dense).max() + 1e-5)


PATH_CASES = [
    # heavier sparsity (tau 0.5, 1-2 kept blocks) so the correction stands well above the
    # bf16 rounding of the output; r picks the device's subspace path
    ("tiny r=16: 32-column subspace", "tiny", dict(kmax=1, tau=0.5), 16, 16),
    ("tiny r=24: whole-matrix Jacobi (d=64)", "tiny", dict(kmax=1, tau=0.5), 16, 24),
    ("medium r=16: 32-column subspace", "medium", dict(H=2, tau=0.5, kmax=2), 4, 16),
    ("medium r=40: 64-column subspace", "medium", dict(H=2, tau=0.5, kmax=2), 4, 40),
    ("medium r=64: whole-matrix Jacobi", "medium", dict(H=2, tau=0.5, kmax=2), 4, 64),
    ("medium r=d: P = I", "medium", dict(H=2, tau=0.5, kmax=2), 4, 128),
]


@pytest.mark.parametrize("desc,name,ov,per_block,r", PATH_CASES, ids=[c[0] for c in PATH_CASES])
def test_probe_correction_itself_on_every_subspace_path(desc, name, ov, per_block, r):
    """The correction o_corr - o_sparse (rows other than the probes) against the oracle's
    want - o_sparse.  The device output is one bf16 rounding of the corrected value, an
    error of at most 2^-9 |o| per element, about |o| 2^-9 / sqrt(3) in rms, while the
    oracle's is exact: the bound is three times that noise relative to the correction, plus
    2 % for the fp32 fit, the bf16 B P of the tensor-core apply and the iterative subspace.
    A wrong subspace or fit is off by order one, a non-finite one fails outright."""
    import block_sparse_attention_33_b200 as sp
    w = get_config(name, **ov)
    Q, K, V, probes, o_sparse, o_corr, status = _run(w, per_block, 100.0, r)
    assert status == sp.OK
    for hi in range(w.H):
        q, k, v = (R.decode_bf16(X[0, hi]) for X in (Q, K, V))
        rows = probes[0, hi].astype(np.int64)
        dense = P.dense_rows(q, k, v, rows)
        want = P.correct(o_sparse[0, hi], dense, rows, 100.0, r)
        keep = np.ones(w.N, bool)
        keep[rows] = False
        got_c = (o_corr[0, hi] - o_sparse[0, hi])[keep]
        want_c = (want - o_sparse[0, hi])[keep]
        assert np.all(np.isfinite(got_c)), hi
        noise = 2.0 ** -9 * np.linalg.norm(o_sparse[0, hi][keep]) / np.sqrt(3.0)
        scale = np.linalg.norm(want_c)
        assert scale > 10 * noise, (hi, scale, noise)   # the case measures something
        rel = np.linalg.norm(got_c - want_c) / scale
        assert rel < 3 * noise / scale + 0.02, (hi, rel, noise / scale)


def test_probe_index_out_of_range_is_flagged():
    import block_sparse_attention_33_b200 as sp
    w = get_config("tiny", kmax=2)
    *_, o_sparse, o_corr, status = _run(w, 4, 100.0, 8, bad_probe=True)
    assert status == sp.ERR_DEVICE
    assert np.isfinite(o_corr).all()


# The composed path against the oracle run on its own: the library's routing,
# routed attention, exact probe rows, ridge fit, subspace and correction on
# one side; oracle.probe_residual.forward_probe (its own routing, its own
# sparse output, its own exact rows) on the other.  Routing may differ only on
# marginal blocks; the corrected outputs must agree within the output bounds
# (every row, or a seeded sample of rows at the Wan-like size).
E2E_CASES = [
    ("tiny d=64, r=16", "tiny", dict(kmax=2), 16, 100.0, 16, 0),
    ("medium 2 heads, r=8", "medium", dict(H=2, tau=0.8), 4, 100.0, 8, 0),
    ("medium 2 heads, r=d", "medium", dict(H=2), 4, 10.0, 128, 0),
    ("wan 2 heads, 384 sampled rows, r=8", "wan", dict(H=2), 1, 100.0, 8, 384),
]


@pytest.mark.parametrize("desc,name,ov,per_block,lam,r,sample", E2E_CASES,
                         ids=[c[0] for c in E2E_CASES])
def test_composed_path_against_oracle_forward_probe(desc, name, ov, per_block, lam, r, sample):
    import torch
    import block_sparse_attention_33_b200 as sp
    from tests.harness import compare_routing, csr_to_kept
    w = get_config(name, **ov)
    Q, K, V = make_qkv(w)
    probes = np.stack([np.stack([probe_rows(w.N, w.b, (6, bi, hi), per_block)
                                 for hi in range(w.H)]) for bi in range(w.B)]).astype(np.int32)
    plan = sp.Plan(w.B, w.H, w.N, w.d, w.b, w.tau, w.kmin, w.kmax, w.residual)
    try:
        q, k, v = to_dev(Q), to_dev(K), to_dev(V)
        o = torch.zeros_like(q)
        row_ptr = torch.zeros(w.B * w.H * plan.nb + 1, dtype=torch.int32, device="cuda")
        col_idx = torch.zeros(max(plan.col_capacity, 1), dtype=torch.int32, device="cuda")
        plan.route(q, k, v, row_ptr, col_idx)
        plan.attend(q, k, v, o)
        plan.probe_correct(q, k, v, o, torch.from_numpy(probes).cuda(), lam, r)
        assert plan.check() == sp.OK
        got = from_dev(o)
        gpu_kept = csr_to_kept(row_ptr.cpu().numpy(), col_idx.cpu().numpy(), w.B, w.H, plan.nb)
    finally:
        plan.close()
    rows = None
    if sample:
        rng = np.random.default_rng(17)
        rows = {(bi, hi): np.sort(np.concatenate([rng.choice(w.N, sample - 8, replace=False),
                                                  probes[bi, hi][:8]]))
                for bi in range(w.B) for hi in range(w.H)}
    ref = P.forward_probe(Q, K, V, w.b, w.tau, w.kmin, w.kmax, w.residual, probes, lam, r,
                          rows=rows)
    bad, marginal, _ = compare_routing(ref["route"], gpu_kept)
    assert bad == 0, f"{bad} non-marginal kept-set disagreements ({marginal} marginal)"
    for bi in range(w.B):
        for hi in range(w.H):
            if rows is None:
                g, want = got[bi, hi], ref["O"][bi, hi]
            else:
                g, want = got[bi, hi][rows[(bi, hi)]], ref["O"][(bi, hi)]
            max_abs, rel = compare_outputs(g, want)
            assert max_abs < MAX_ABS and rel < REL_L2, (bi, hi, max_abs, rel, marginal)
