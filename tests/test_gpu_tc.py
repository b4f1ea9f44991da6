"""The tcgen05/TMEM attention kernel (128-token blocks) against the oracle and
against the independent warp-MMA kernel on the same inputs and CSR."""
import os

import numpy as np
import pytest

from tests.harness import MAX_ABS, REL_L2, compare_outputs, oracle_check, run_library
from workloads import get_config, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu(gpu_required):
    import block_sparse_attention_33_b200 as sp
    sp.lib()


def run_with(kernel, w, Q, K, V, **kw):
    old = os.environ.get("SPATTN_ATTN")
    try:
        if kernel == "mma":
            os.environ["SPATTN_ATTN"] = "mma"
        else:
            os.environ.pop("SPATTN_ATTN", None)
        return run_library(w, Q, K, V, **kw)
    finally:
        if old is None:
            os.environ.pop("SPATTN_ATTN", None)
        else:
            os.environ["SPATTN_ATTN"] = old


SMALL = [
    ("one block, d=128", dict(grid=(1, 1, 128), d=128, b=128, H=1, kmax=4)),
    ("4 blocks, d=128", dict(grid=(1, 4, 128), d=128, b=128, H=1, kmax=4, tau=0.7)),
    ("partial tail, d=128", dict(grid=(1, 5, 100), d=128, b=128, H=2, kmax=8, tau=0.8)),
    ("d=64 b=128", dict(grid=(2, 8, 64), d=64, b=128, H=2, tau=0.85)),
    ("no residual", dict(grid=(2, 8, 64), d=128, b=128, H=2, tau=0.6, residual=0)),
    ("tau=1 dense", dict(grid=(2, 8, 64), d=128, b=128, H=2, tau=1.0)),
    # 64-token blocks: two query blocks per 128-row tile, two key blocks per
    # key tile (union of the two kept sets)
    ("b=64 d=64", dict()),
    ("b=64 d=128", dict(d=128, H=2, tau=0.8)),
    ("b=64 no residual", dict(residual=0, kmax=3, tau=0.6)),
    ("b=64 odd nb, one token in the last block", dict(grid=(1, 5, 13), kmax=2)),
    ("b=64 three blocks, last tile single", dict(grid=(1, 3, 64), kmax=2, tau=0.5)),
    ("b=64 partial last block of 20", dict(grid=(1, 7, 12), d=128, kmax=3, tau=0.7)),
]


@pytest.mark.parametrize("desc,ov", SMALL, ids=[s[0] for s in SMALL])
def test_tc_small_against_oracle_and_mma(desc, ov):
    w = get_config("tiny", **ov)
    Q, K, V = make_qkv(w)
    res = run_with("tc", w, Q, K, V)
    assert res["status"] == 0
    fig = oracle_check(w, Q, K, V, res)
    assert fig["bad"] == 0, fig
    assert fig["max_abs"] < MAX_ABS and fig["rel_l2"] < REL_L2, fig
    ref = run_with("mma", w, Q, K, V)
    assert np.array_equal(ref["row_ptr"], res["row_ptr"])
    max_abs, rel = compare_outputs(res["O"], ref["O"])
    assert max_abs < MAX_ABS and rel < REL_L2, (max_abs, rel)


@pytest.mark.parametrize("residual", [1, 0])
def test_tc_medium(residual):
    w = get_config("medium", residual=residual)
    Q, K, V = make_qkv(w)
    res = run_with("tc", w, Q, K, V)
    assert res["status"] == 0
    fig = oracle_check(w, Q, K, V, res)
    assert fig["bad"] == 0 and fig["max_abs"] < MAX_ABS and fig["rel_l2"] < REL_L2, fig


def test_tc_hilbert_stress_shape_small():
    w = get_config("stress", H=2)
    Q, K, V = make_qkv(w)
    import block_sparse_attention_33_b200 as sp
    perm = sp.spattn_hilbert_perm(*w.grid)
    res = run_with("tc", w, Q, K, V, perm=perm)
    assert res["status"] == 0
    rows = {(0, h): np.arange(0, w.N, 97) for h in range(w.H)}
    fig = oracle_check(w, Q, K, V, res, perm=perm, rows={k: perm[v] for k, v in rows.items()})
    assert fig["bad"] == 0 and fig["max_abs"] < MAX_ABS and fig["rel_l2"] < REL_L2, fig


# ---- the persistent work loop: more items than SMs, items without tasks,
# ---- the self-resetting work counter

def _oracle_csr(w, Q, K, V):
    from oracle import spattn_ref as R
    from tests.harness import kept_to_csr
    ref = R.forward(Q, K, V, w.b, w.tau, w.kmin, w.kmax, w.residual, want_output=False)
    return {key: [np.asarray(x) for x in r["kept"]] for key, r in ref["route"].items()}


def test_tc_caller_csr_with_empty_rows_on_unrouted_workspace():
    """Caller CSR in which every 5th query block keeps nothing, no residual
    (those items have no tasks and must come out as zeros), on a workspace
    that was never routed and holds garbage: the attention call clears its
    own work counter.  256 items, more than the SMs, so CTAs loop."""
    import torch
    import block_sparse_attention_33_b200 as sp
    from oracle import spattn_ref as R
    from tests.harness import from_dev, kept_to_csr, to_dev
    w = get_config("medium", H=4, residual=0, tau=0.7)
    Q, K, V = make_qkv(w)
    kept = _oracle_csr(w, Q, K, V)
    empty = {(0, h): [i for i in range(w.nb) if (i + h) % 5 == 0] for h in range(w.H)}
    for key, blocks in empty.items():
        for i in blocks:
            kept[key][i] = np.zeros(0, np.int64)
    rp, ci = kept_to_csr(kept, w.B, w.H, w.nb)
    plan = sp.Plan(w.B, w.H, w.N, w.d, w.b, w.tau, w.kmin, w.kmax, w.residual)
    try:
        plan.workspace.fill_(0x7F)                       # never routed: garbage control words
        q, k, v = to_dev(Q), to_dev(K), to_dev(V)
        o = torch.full_like(q, 3.0)
        plan.attend(q, k, v, o, torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda())
        assert plan.check() == 0
        O = from_dev(o)
    finally:
        plan.close()
    b = w.b
    rows = {}
    for h in range(w.H):
        keep_blocks = [i for i in range(w.nb) if (i + h) % 5 != 0]
        rows[(0, h)] = np.concatenate([np.arange(i * b, i * b + b, 7) for i in keep_blocks])
        for i in empty[(0, h)]:
            assert np.all(O[0, h, i * b:(i + 1) * b] == 0.0), (h, i)
    ref = R.forward(Q, K, V, w.b, w.tau, w.kmin, w.kmax, w.residual, rows=rows, kept_override=kept)
    got = np.concatenate([O[0, h, rows[(0, h)]] for h in range(w.H)])
    want = np.concatenate([ref["O"][(0, h)] for h in range(w.H)])
    max_abs, rel = compare_outputs(got, want)
    assert max_abs < MAX_ABS and rel < REL_L2, (max_abs, rel)


def test_tc_repeated_attend_is_bitwise_stable():
    """Three attention calls after one routing call: the work counter resets
    itself at the end of each launch, and an item's output does not depend on
    which CTA ran it."""
    import torch
    import block_sparse_attention_33_b200 as sp
    from tests.harness import to_dev
    w = get_config("medium", H=4)
    Q, K, V = make_qkv(w)
    plan = sp.Plan(w.B, w.H, w.N, w.d, w.b, w.tau, w.kmin, w.kmax, w.residual)
    try:
        q, k, v = to_dev(Q), to_dev(K), to_dev(V)
        plan.route(q, k, v)
        outs = []
        for _ in range(3):
            o = torch.zeros_like(q)
            plan.attend(q, k, v, o)
            outs.append(o)
        assert plan.check() == 0
        torch.cuda.synchronize()
    finally:
        plan.close()
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    assert torch.equal(outs[0].view(torch.int16), outs[2].view(torch.int16))


def test_tc_routing_reuse_across_calls():
    """Route once on inputs A, then pool + attend inputs B: the output is the
    oracle's attention of B over A's kept sets (B's own means feed the
    residual).  With the Hilbert permutation, so the pooling's permuted
    copies of B are what the attention reads."""
    import torch
    import block_sparse_attention_33_b200 as sp
    from oracle import spattn_ref as R
    from tests.harness import csr_to_kept, from_dev, to_dev
    w = get_config("medium", H=2, tau=0.8)
    wb = w.with_(seed=w.seed + 77)
    QA, KA, VA = make_qkv(w)
    QB, KB, VB = make_qkv(wb)
    perm = sp.spattn_hilbert_perm(*w.grid)
    plan = sp.Plan(w.B, w.H, w.N, w.d, w.b, w.tau, w.kmin, w.kmax, w.residual, perm)
    try:
        rows = w.B * w.H * plan.nb
        rp = torch.zeros(rows + 1, dtype=torch.int32, device="cuda")
        ci = torch.zeros(max(plan.col_capacity, 1), dtype=torch.int32, device="cuda")
        qa, ka, va = to_dev(QA), to_dev(KA), to_dev(VA)
        plan.route(qa, ka, va, rp, ci)
        qb, kb, vb = to_dev(QB), to_dev(KB), to_dev(VB)
        o = torch.zeros_like(qb)
        plan.pool(qb, kb, vb)
        plan.attend(qb, kb, vb, o)
        assert plan.check() == 0
        O = from_dev(o)
        kept_a = csr_to_kept(rp.cpu().numpy(), ci.cpu().numpy(), w.B, w.H, plan.nb)
    finally:
        plan.close()
    pick = {(0, h): perm[np.arange(0, w.N, 53)] for h in range(w.H)}
    ref = R.forward(QB, KB, VB, w.b, w.tau, w.kmin, w.kmax, w.residual, perm=perm, rows=pick,
                    kept_override=kept_a)
    got = np.concatenate([O[0, h, pick[(0, h)]] for h in range(w.H)])
    want = np.concatenate([ref["O"][(0, h)] for h in range(w.H)])
    max_abs, rel = compare_outputs(got, want)
    assert max_abs < MAX_ABS and rel < REL_L2, (max_abs, rel)
    # and it differs from B's own routing's result somewhere (A's sets are not B's)
    own = R.forward(QB, KB, VB, w.b, w.tau, w.kmin, w.kmax, w.residual, perm=perm, rows=pick)
    assert any(not np.array_equal(np.sort(a), np.sort(b))
               for key in own["route"] for a, b in zip(own["route"][key]["kept"], kept_a[key]))


@pytest.mark.parametrize("perm_on", [False, True])
def test_writes_stay_inside_workspace_and_output(perm_on):
    """Canary bytes before and after the workspace and the output tensor are
    untouched by a full forward (pool, routing, attention; with the Hilbert
    permutation the pooling also writes the permuted copies)."""
    import torch
    import block_sparse_attention_33_b200 as sp
    from tests.harness import to_dev
    w = get_config("medium", H=2, tau=0.8)
    Q, K, V = make_qkv(w)
    perm = sp.spattn_hilbert_perm(*w.grid) if perm_on else None
    plan = sp.Plan(w.B, w.H, w.N, w.d, w.b, w.tau, w.kmin, w.kmax, w.residual, perm)
    pad = 1 << 20
    try:
        ws = torch.full((plan.ws_bytes + 2 * pad,), 0xA5, dtype=torch.uint8, device="cuda")
        plan.workspace = ws[pad:pad + plan.ws_bytes]
        q, k, v = to_dev(Q), to_dev(K), to_dev(V)
        n = q.numel()
        ob = torch.full((n + 2 * (pad // 2),), 7.0, dtype=torch.bfloat16, device="cuda")
        o = ob[pad // 2:pad // 2 + n].view(q.shape)
        plan.forward(q, k, v, o)
        assert plan.check() == 0
        torch.cuda.synchronize()
        assert torch.all(ws[:pad] == 0xA5) and torch.all(ws[pad + plan.ws_bytes:] == 0xA5)
        assert torch.all(ob[:pad // 2] == 7.0) and torch.all(ob[pad // 2 + n:] == 7.0)
        assert torch.isfinite(o.float()).all()
    finally:
        plan.close()
