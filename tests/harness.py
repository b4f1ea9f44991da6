"""Helpers shared by the GPU parity tests: run the library, compare with the oracle."""
from __future__ import annotations

import numpy as np

import oracle
from oracle import spattn_ref as R

# Acceptance bounds for outputs (bf16 output of a bf16-input attention vs the
# fp64 oracle): element-wise max-abs and relative L2 over the compared rows.
MAX_ABS = 2e-2
REL_L2 = 4e-3


def to_dev(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def from_dev(t) -> np.ndarray:
    """bf16 device tensor -> float64 numpy (exact widening)."""
    return t.float().cpu().numpy().astype(np.float64)


def run_library(w, Q, K, V, perm=None, kept_csr=None, want_means=False, tau=None, routing=0):
    """Run route + attend through the C ABI; returns dict with O (fp64), CSR, means.
    routing: 0 centroid estimate, 1 PAMA, optionally | SELECT_THRESHOLD."""
    import torch
    import block_sparse_attention_33_b200 as sp
    tau = w.tau if tau is None else tau
    B, H, N, d = Q.shape
    plan = sp.Plan(B, H, N, d, w.b, tau, w.kmin, w.kmax, w.residual, perm, routing=routing)
    try:
        q, k, v = to_dev(Q), to_dev(K), to_dev(V)
        o = torch.zeros_like(q)
        rows = B * H * plan.nb
        row_ptr = torch.zeros(rows + 1, dtype=torch.int32, device="cuda")
        col_idx = torch.full((max(plan.col_capacity, 1),), -7, dtype=torch.int32, device="cuda")
        plan.route(q, k, v, row_ptr, col_idx)
        if kept_csr is None:
            plan.attend(q, k, v, o)
        else:
            rp, ci = kept_csr
            plan.attend(q, k, v, o, torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda())
        out = {"nb": plan.nb}
        if want_means:
            shape = (B, H, plan.nb, d)
            bars = [torch.empty(shape, dtype=torch.float32, device="cuda") for _ in range(3)]
            sp.spattn_means(plan.handle, plan.workspace, *bars)
            out["means"] = [x.cpu().numpy().astype(np.float64) for x in bars]
        status = plan.check()
        torch.cuda.synchronize()
        out["status"] = status
        out["O"] = from_dev(o)
        out["row_ptr"] = row_ptr.cpu().numpy()
        out["col_idx"] = col_idx.cpu().numpy()
        return out
    finally:
        plan.close()


def csr_to_kept(row_ptr, col_idx, B, H, nb):
    kept = {}
    for bi in range(B):
        for hi in range(H):
            rows = []
            for i in range(nb):
                r = (bi * H + hi) * nb + i
                rows.append(col_idx[row_ptr[r]:row_ptr[r + 1]].astype(np.int64))
            kept[(bi, hi)] = rows
    return kept


def kept_to_csr(kept, B, H, nb):
    rp, ci = [0], []
    for bi in range(B):
        for hi in range(H):
            for i in range(nb):
                ks = np.asarray(kept[(bi, hi)][i], dtype=np.int32)
                ci.extend(ks.tolist())
                rp.append(rp[-1] + len(ks))
    return np.asarray(rp, np.int32), np.asarray(ci if ci else [0], np.int32)


def compare_routing(routes, gpu_kept):
    """Count kept-set disagreements: (non-marginal, marginal, rows differing).

    A disagreement on a block that the oracle marks marginal (cumulative-mass
    margin to tau below 1e-4, or a near-tie at the cut) is allowed and
    counted; any other disagreement is a failure.
    """
    bad = marg = rows = 0
    for key, r in routes.items():
        for i, ok in enumerate(r["kept"]):
            g = gpu_kept[key][i]
            if not np.all(np.diff(g) > 0):
                bad += 1          # not strictly ascending
                continue
            diff = np.setxor1d(ok, g)
            if len(diff):
                rows += 1
                m = np.isin(diff, r["marginal"][i])
                marg += int(m.sum())
                bad += int((~m).sum())
    return bad, marg, rows


def compare_outputs(got: np.ndarray, ref: np.ndarray):
    err = got - ref
    max_abs = float(np.max(np.abs(err))) if err.size else 0.0
    den = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(err) / den) if den > 0 else float(np.linalg.norm(err))
    return max_abs, rel


def oracle_check(w, Q, K, V, res, perm=None, rows=None, tau=None, routing="centroid",
                 selection="top_p"):
    """Oracle routing vs the library CSR, then oracle attention on the library's
    kept sets vs the library output.  Returns a dict of figures."""
    tau = w.tau if tau is None else tau
    B, H, N, d = Q.shape
    nb = res["nb"]
    gpu_kept = csr_to_kept(res["row_ptr"], res["col_idx"], B, H, nb)
    ref = R.forward(Q, K, V, w.b, tau, w.kmin, w.kmax, w.residual, perm=perm, rows=rows,
                    kept_override=gpu_kept, routing=routing, selection=selection)
    bad, marg, nrows = compare_routing(ref["route"], gpu_kept)
    if rows is None:
        max_abs, rel = compare_outputs(res["O"], ref["O"])
    else:
        got = np.concatenate([res["O"][bi, hi, rows[(bi, hi)]] for (bi, hi) in rows])
        want = np.concatenate([ref["O"][(bi, hi)] for (bi, hi) in rows])
        max_abs, rel = compare_outputs(got, want)
    kept_total = sum(len(x) for v in gpu_kept.values() for x in v)
    return {"bad": bad, "marginal": marg, "rows_diff": nrows, "max_abs": max_abs, "rel_l2": rel,
            "ref": ref, "kept_fraction": kept_total / (B * H * nb * nb)}
