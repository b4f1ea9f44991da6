"""Routed block-sparse attention, plain fp64 reference (test infrastructure only).

Notation: Q, K, V are [B, H, N, d]; tokens are cut into nb = ceil(N/b) blocks
of b tokens, block j holding n_j tokens (only the last block may be partial).
Query blocks use the same partition as key blocks.

Readings of points the pages leave open:

* natural logarithm in the ln n_j term; scale 1/sqrt(d) on every logit, the
  proxy and the pseudo-keys alike;
* the Top-p rule of PARK page 3.2 (blocks taken in descending estimated
  importance while the accumulated estimate is below the threshold) is read
  as: order blocks by p descending, ties to the lower block index, and
  keep rank r iff the mass of the ranks before it is < tau; so the kept count
  k* is the length of the shortest prefix whose mass is >= tau;
* tau >= 1 keeps every block (no prefix shorter than nb is needed, and
  rounding must not drop a block), tau <= 0 gives k* = 0;
* the budget is k = min(max(k*, kmin), kmax, nb);
* the on-the-fly block thresholding of the Sol-Attn abstract (a block is
  critical when its proxy score passes a threshold; no proxy map is stored)
  is read as a fixed threshold on the block probability, p_ij >= theta,
  with the same clamp and the same order (p descending, ties to the lower
  index) when a clamp binds (route_threshold);
* the partial last query block is routed from its own mean over n_i tokens;
* the pseudo-key of a dropped block j uses the per-token query q (not the
  block mean): logit q . Kbar_j / sqrt(d) + ln n_j, value Vbar_j;
* a permutation perm is a gather: Xp[n] = X[perm[n]]; the output is
  scattered back with O[perm[n]] = Op[n].
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

# Kept-set comparison margins.  A block whose cumulative-mass margin
# |E_rank - tau| is below MASS_MARGIN may legitimately flip between two
# correct implementations working in different precisions; so may a block
# at the cut whose probability ties, within a relative TIE_MARGIN, with the
# block on the other side of the cut.
MASS_MARGIN = 1e-4
TIE_MARGIN = 1e-4


# ---------------------------------------------------------------- inputs ---

def decode_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly.

    A bf16 value is the upper half of an IEEE binary32 word: sign, 8 exponent
    bits, 7 mantissa bits.  Written out from that definition.
    """
    u = np.asarray(bits, dtype=np.uint16).astype(np.int64)
    sign = np.where((u >> 15) & 1, -1.0, 1.0)
    exp = (u >> 7) & 0xFF
    man = (u & 0x7F).astype(np.float64)
    normal = sign * np.ldexp(1.0 + man / 128.0, (exp - 127).astype(np.int64))
    subnormal = sign * np.ldexp(man / 128.0, -126)
    out = np.where(exp == 0, subnormal, normal)
    out = np.where(exp == 0xFF, np.where(man == 0, sign * np.inf, np.nan), out)
    return out


def block_sizes(N: int, b: int) -> np.ndarray:
    """n_j for j = 0..nb-1: b everywhere except a possibly partial last block."""
    nb = -(-N // b)
    n = np.full(nb, b, dtype=np.int64)
    n[-1] = N - (nb - 1) * b
    return n


def gather_tokens(X: np.ndarray, perm: Optional[np.ndarray]) -> np.ndarray:
    """Xp[..., n, :] = X[..., perm[n], :] (identity when perm is None)."""
    return X if perm is None else X[..., np.asarray(perm), :]


def scatter_tokens(Xp: np.ndarray, perm: Optional[np.ndarray]) -> np.ndarray:
    """Inverse of gather_tokens: X[..., perm[n], :] = Xp[..., n, :]."""
    if perm is None:
        return Xp
    X = np.empty_like(Xp)
    X[..., np.asarray(perm), :] = Xp
    return X


# --------------------------------------------------------------- pooling ---

def block_means(X: np.ndarray, b: int) -> np.ndarray:
    """Block means over the token axis: [..., N, d] -> [..., nb, d] (fp64).

    Blocks are represented by the average of their tokens (PARK page,
    abstract: query and key blocks are compared through their averages).
    """
    N = X.shape[-2]
    n = block_sizes(N, b)
    out = np.empty(X.shape[:-2] + (len(n), X.shape[-1]), dtype=np.float64)
    for j in range(len(n)):
        out[..., j, :] = X[..., j * b: j * b + n[j], :].sum(axis=-2) / n[j]
    return out


# --------------------------------------------------------------- scoring ---

def proxy_logits(Qbar: np.ndarray, Kbar: np.ndarray, n: np.ndarray) -> np.ndarray:
    """s_ij = Qbar_i . Kbar_j / sqrt(d) + ln n_j for one head: [nb, nb].

    The ln n_j term makes s_ij the centroid lower bound on the exact block
    log-mass ln sum_{k in j} exp(q . k / sqrt(d)) (PARK page section D.2,
    Jensen's inequality), evaluated at the block-mean query.
    """
    d = Qbar.shape[-1]
    return (Qbar @ Kbar.T) / math.sqrt(d) + np.log(n.astype(np.float64))[None, :]


def block_softmax(s: np.ndarray) -> np.ndarray:
    """p_ij = softmax over j of s_ij, max-subtracted, fp64."""
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=-1, keepdims=True)


def pama_importance(q: np.ndarray, Kbar: np.ndarray, n: np.ndarray) -> np.ndarray:
    """Block importance of one query block by per-query attention-mass
    aggregation (PARK page 5.1, PAMA): every query token q keeps its own
    softmax over the key blocks of the centroid logit q . Kbar_j / sqrt(d) +
    ln n_j (the same block log-mass estimate as the proxy), and the block's
    importance row is the mean of its tokens' rows (PARK page 3.2: the
    average attention weight the block's queries give each key block).
    q: [n_i, d] tokens of the query block; returns p_i [nb], summing to 1."""
    d = q.shape[-1]
    s = q @ Kbar.T / math.sqrt(d) + np.log(n.astype(np.float64))[None, :]
    return block_softmax(s).mean(axis=0)


def exact_block_logmass(q: np.ndarray, Kblock: np.ndarray) -> float:
    """ln sum_{k in block} exp(q . k / sqrt(d)): the quantity s_ij bounds."""
    z = Kblock @ q / math.sqrt(q.shape[-1])
    m = z.max()
    return float(m + math.log(np.exp(z - m).sum()))


# --------------------------------------------------------------- routing ---

def route_rows(p: np.ndarray, tau: float, kmin: int, kmax: int):
    """Top-p block selection for every query block of one head.

    p: [nb_q, nb] block probabilities.  Returns a dict with
      kept      list of int arrays, ascending block index, one per row
      k         int array of budgets
      marginal  list of int arrays: blocks whose decision sits within the
                comparison margins (see MASS_MARGIN / TIE_MARGIN)
      E         [nb_q, nb] exclusive prefix mass at each block's rank
    """
    nq, nb = p.shape
    kept, ks, marginal = [], np.empty(nq, np.int64), []
    E_all = np.empty_like(p)
    idx = np.arange(nb)
    kcap = min(kmax, nb)
    for i in range(nq):
        row = p[i]
        # descending probability, ties broken by the lower block index
        order = np.lexsort((idx, -row))
        sorted_p = row[order]
        E = np.concatenate(([0.0], np.cumsum(sorted_p)[:-1]))
        if tau >= 1.0:
            kstar = nb
        else:
            kstar = int(np.count_nonzero(E < tau))  # E is non-decreasing
        k = min(max(kstar, kmin), kcap)
        ks[i] = k
        kept.append(np.sort(order[:k]))
        E_rank = np.empty(nb)
        E_rank[order] = E
        E_all[i] = E_rank
        marg = set()
        if 0.0 < tau < 1.0 and kmin <= kstar <= kcap:
            # the cut was set by the mass rule: blocks close to tau
            marg.update(np.nonzero(np.abs(E_rank - tau) < MASS_MARGIN)[0].tolist())
        if 0 < k < nb:
            p_in, p_out = sorted_p[k - 1], sorted_p[k]
            # kept blocks tying with the first dropped one
            r_in = np.nonzero(sorted_p[:k] - p_out <= TIE_MARGIN * sorted_p[:k])[0]
            # dropped blocks tying with the last kept one
            r_out = k + np.nonzero(p_in - sorted_p[k:] <= TIE_MARGIN * p_in)[0]
            marg.update(order[r_in].tolist())
            marg.update(order[r_out].tolist())
        marginal.append(np.array(sorted(marg), dtype=np.int64))
    return {"kept": kept, "k": ks, "marginal": marginal, "E": E_all}


def route_threshold(p: np.ndarray, theta: float, kmin: int, kmax: int):
    """Per-block probability threshold (Sol-Attn abstract: on-the-fly block
    thresholding of the proxy scores, dynamic but controllable budgets).

    Reading: block j of query row i is critical iff p_ij >= theta; the
    budget is clamped to [kmin, min(kmax, nb)] by taking blocks in the same
    order as the Top-p rule (p descending, ties to the lower index).  The
    critical set is a prefix of that order, so no sort is needed unless a
    clamp binds.  Returns the same dict as route_rows (E: exclusive prefix
    mass at each block's rank); marginal blocks are those whose p lies
    within a relative TIE_MARGIN of theta, plus, when a clamp set the cut,
    the near-ties across the cut."""
    nq, nb = p.shape
    kept, ks, marginal = [], np.empty(nq, np.int64), []
    E_all = np.empty_like(p)
    idx = np.arange(nb)
    kcap = min(kmax, nb)
    for i in range(nq):
        row = p[i]
        crit = np.nonzero(row >= theta)[0]
        kstar = len(crit)
        order = np.lexsort((idx, -row))
        sorted_p = row[order]
        k = min(max(kstar, kmin), kcap)
        ks[i] = k
        kept.append(np.sort(order[:k]) if k != kstar else crit)
        E = np.concatenate(([0.0], np.cumsum(sorted_p)[:-1]))
        E_rank = np.empty(nb)
        E_rank[order] = E
        E_all[i] = E_rank
        marg = set()
        if k == kstar:
            marg.update(np.nonzero(np.abs(row - theta) <= TIE_MARGIN * abs(theta))[0].tolist())
        elif 0 < k < nb:
            p_in, p_out = sorted_p[k - 1], sorted_p[k]
            r_in = np.nonzero(sorted_p[:k] - p_out <= TIE_MARGIN * sorted_p[:k])[0]
            r_out = k + np.nonzero(p_in - sorted_p[k:] <= TIE_MARGIN * p_in)[0]
            marg.update(order[r_in].tolist())
            marg.update(order[r_out].tolist())
        marginal.append(np.array(sorted(marg), dtype=np.int64))
    return {"kept": kept, "k": ks, "marginal": marginal, "E": E_all}


# ------------------------------------------------------------- attention ---

def attend_block(q: np.ndarray, Kp: np.ndarray, Vp: np.ndarray, kept: Sequence[int],
                 n: np.ndarray, b: int, residual: bool,
                 Kbar: Optional[np.ndarray] = None,
                 Vbar: Optional[np.ndarray] = None) -> np.ndarray:
    """Outputs for query tokens q [r, d] of one query block, one head.

    Each token's logit set is {q . k / sqrt(d) : k a token of a kept block};
    in residual mode it also holds, for every dropped block j, the pseudo-key
    q . Kbar_j / sqrt(d) + ln n_j with value Vbar_j.  One softmax over that
    set (max, then sum), output sum(w v) / sum(w).
    """
    d = q.shape[-1]
    nb = len(n)
    kept = np.asarray(sorted(int(j) for j in kept), dtype=np.int64)
    toks = np.concatenate([np.arange(j * b, j * b + n[j]) for j in kept]) if len(kept) else \
        np.zeros(0, np.int64)
    logits = [q @ Kp[toks].T / math.sqrt(d)]
    values = [Vp[toks]]
    if residual:
        dropped = np.setdiff1d(np.arange(nb), kept)
        if len(dropped):
            logits.append(q @ Kbar[dropped].T / math.sqrt(d)
                          + np.log(n[dropped].astype(np.float64))[None, :])
            values.append(Vbar[dropped])
    z = np.concatenate(logits, axis=1)
    vals = np.concatenate(values, axis=0)
    m = z.max(axis=1, keepdims=True)
    w = np.exp(z - m)
    return (w @ vals) / w.sum(axis=1, keepdims=True)


def attention(Qp, Kp, Vp, kept_rows, b: int, residual: bool, Kbar=None, Vbar=None,
              rows: Optional[np.ndarray] = None) -> np.ndarray:
    """Routed attention for one head in the blocked (possibly permuted) order.

    kept_rows[i] is the kept block set of query block i.  If ``rows`` is given,
    only those token rows are computed and returned ([len(rows), d]);
    otherwise all N rows are returned.
    """
    N, d = Qp.shape
    n = block_sizes(N, b)
    want = np.arange(N) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.empty((len(want), d))
    blk = want // b
    for i in np.unique(blk):
        sel = np.nonzero(blk == i)[0]
        out[sel] = attend_block(Qp[want[sel]], Kp, Vp, kept_rows[i], n, b, residual,
                                Kbar, Vbar)
    return out


def attention_flops(kept_rows, n: np.ndarray, residual: bool, d: int) -> tuple:
    """(exact-token FLOPs, residual FLOPs) of one head: 4 d per (query, key) pair."""
    nb = len(n)
    exact = 0
    res = 0
    for i, ks in enumerate(kept_rows):
        nk = int(n[np.asarray(ks, dtype=np.int64)].sum())
        exact += int(n[i]) * nk
        if residual:
            res += int(n[i]) * (nb - len(ks))
    return 4 * d * exact, 4 * d * res


# ------------------------------------------------------------ full chain ---

def forward(Q, K, V, b: int, tau: float, kmin: int, kmax: int, residual: int,
            perm: Optional[np.ndarray] = None, rows: Optional[dict] = None,
            kept_override: Optional[dict] = None, want_output: bool = True,
            routing: str = "centroid", selection: str = "top_p"):
    """The whole path for bf16 inputs Q, K, V ([B, H, N, d] uint16 bits).

    rows:          optional {(b, h): array of token indices in the ORIGINAL
                   order} -- only those outputs are computed (for large sizes).
    kept_override: optional {(b, h): list of kept sets} to run the attention
                   with externally supplied kept sets (routing is still
                   computed and returned).
    routing:       "centroid" (p from the block-mean proxy) or "pama" (p from
                   pama_importance of each query block's tokens).
    selection:     "top_p" (route_rows, tau is the mass threshold) or
                   "threshold" (route_threshold, tau is read as the per-block
                   probability threshold theta).
    Returns a dict with Qbar/Kbar/Vbar (fp64 [B,H,nb,d]), route (per (b,h)
    route_rows results), and O: either [B,H,N,d] fp64 or {(b,h): [r, d]}.
    """
    B, H, N, d = Q.shape
    n = block_sizes(N, b)
    perm = None if perm is None else np.asarray(perm, dtype=np.int64)
    inv = None
    if perm is not None:
        inv = np.empty_like(perm)
        inv[perm] = np.arange(N)
    Qbar = np.empty((B, H, len(n), d))
    Kbar = np.empty_like(Qbar)
    Vbar = np.empty_like(Qbar)
    routes = {}
    O = np.empty((B, H, N, d)) if (rows is None and want_output) else {}
    for bi in range(B):
        for hi in range(H):
            q = gather_tokens(decode_bf16(Q[bi, hi]), perm)
            k = gather_tokens(decode_bf16(K[bi, hi]), perm)
            v = gather_tokens(decode_bf16(V[bi, hi]), perm)
            Qbar[bi, hi] = block_means(q, b)
            Kbar[bi, hi] = block_means(k, b)
            Vbar[bi, hi] = block_means(v, b)
            if routing == "pama":
                starts = np.concatenate([[0], np.cumsum(n)[:-1]])
                p = np.stack([pama_importance(q[s0:s0 + nj], Kbar[bi, hi], n)
                              for s0, nj in zip(starts, n)])
            else:
                p = block_softmax(proxy_logits(Qbar[bi, hi], Kbar[bi, hi], n))
            if selection == "threshold":
                r = route_threshold(p, tau, kmin, kmax)
            elif selection == "top_p":
                r = route_rows(p, tau, kmin, kmax)
            else:
                raise ValueError(f"selection must be 'top_p' or 'threshold', got {selection!r}")
            r["p"] = p
            routes[(bi, hi)] = r
            if not want_output:
                continue
            kept = r["kept"] if kept_override is None else kept_override[(bi, hi)]
            if rows is None:
                Op = attention(q, k, v, kept, b, bool(residual), Kbar[bi, hi], Vbar[bi, hi])
                O[bi, hi] = scatter_tokens(Op, perm)
            else:
                orig = np.asarray(rows[(bi, hi)], dtype=np.int64)
                blocked = orig if inv is None else inv[orig]
                O[(bi, hi)] = attention(q, k, v, kept, b, bool(residual),
                                        Kbar[bi, hi], Vbar[bi, hi], rows=blocked)
    return {"Qbar": Qbar, "Kbar": Kbar, "Vbar": Vbar, "route": routes, "O": O, "n": n}
