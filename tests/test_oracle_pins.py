"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each test ties one oracle step to a closed form, a library routine (torch
fp64), brute-force enumeration, or an invariant the pages state, so that a
plausible slip (a dropped ln n_j, a wrong scale, a transposed product, an
inclusive instead of exclusive prefix, a wrong tie-break, a residual built
from the block-mean query) fails at least one of them.
"""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import spattn_ref as R
from workloads import get_config, make_qkv, f32_to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def sdpa64(q, k, v, mask=None):
    """Library softmax attention in fp64 (torch), q/k/v [N, d] numpy."""
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64))[None, None]
    out = torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), attn_mask=None if mask is None else torch.from_numpy(mask)[None, None])
    return out[0, 0].numpy()


def rand_bf16(rng, shape, scale=1.0):
    return f32_to_bf16_bits((rng.standard_normal(shape) * scale).astype(np.float32))


# ------------------------------------------------------------ bf16 decode --

def test_decode_bf16_matches_torch_for_every_pattern():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = R.decode_bf16(bits)
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


# -------------------------------------------------------------- partition --

def test_block_partition_matches_workload_definitions():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "block_partition.txt"))
            if l.strip() and not l.startswith("#")]
    assert len(rows) == 5
    for name, T, Hs, W, b, N, nb, nlast in rows:
        w = get_config(name)
        assert w.grid == (int(T), int(Hs), int(W)) and w.b == int(b)
        assert w.N == int(N)
        n = R.block_sizes(w.N, w.b)
        assert len(n) == int(nb) and n[-1] == int(nlast) and n.sum() == w.N


# ---------------------------------------------------------------- pooling --

def test_block_means_closed_forms():
    N, b, d = 300, 64, 3  # last block partial: 300 = 4*64 + 44
    t = np.arange(N, dtype=np.float64)
    X = np.stack([t, np.full(N, 7.0), (t % b) ** 2], axis=1)
    m = R.block_means(X, b)
    n = R.block_sizes(N, b)
    for j in range(len(n)):
        lo, cnt = j * b, n[j]
        assert m[j, 0] == lo + (cnt - 1) / 2          # mean of lo..lo+cnt-1
        assert m[j, 1] == 7.0
        assert m[j, 2] == pytest.approx((cnt - 1) * (2 * cnt - 1) / 6, rel=1e-15)
    assert n[-1] == 44


# ---------------------------------------------------------------- scoring --

def test_proxy_equals_block_logmass_for_constant_blocks():
    """Constant query block + constant key block: the centroid estimate is the
    exact block log-mass (PARK page D.1/D.2: identical queries make the query
    side exact; equal scores make Jensen's bound tight)."""
    rng = np.random.default_rng(1)
    d, b, nb = 16, 8, 5
    N = b * nb - 3                       # partial last block
    qrows = np.repeat(rng.standard_normal((nb, d)), b, axis=0)[:N]
    krows = np.repeat(rng.standard_normal((nb, d)) * 2, b, axis=0)[:N]
    n = R.block_sizes(N, b)
    s = R.proxy_logits(R.block_means(qrows, b), R.block_means(krows, b), n)
    for i in range(nb):
        for j in range(nb):
            blk = torch.from_numpy(krows[j * b: j * b + n[j]])
            exact = torch.logsumexp(blk @ torch.from_numpy(qrows[i * b]) / math.sqrt(d), 0).item()
            assert s[i, j] == pytest.approx(exact, abs=1e-12)


def test_proxy_is_jensen_lower_bound():
    """PARK page D.2: the centroid estimate lower-bounds the exact block log-mass."""
    rng = np.random.default_rng(2)
    d, b, nb = 32, 16, 6
    N = b * nb
    qrows = np.repeat(rng.standard_normal((nb, d)), b, axis=0)   # Qbar_i = q
    krows = rng.standard_normal((N, d)) * 1.5
    n = R.block_sizes(N, b)
    s = R.proxy_logits(R.block_means(qrows, b), R.block_means(krows, b), n)
    for i in range(nb):
        q = torch.from_numpy(qrows[i * b])
        for j in range(nb):
            exact = torch.logsumexp(torch.from_numpy(krows[j * b:(j + 1) * b]) @ q / math.sqrt(d), 0)
            assert s[i, j] < exact.item()


def test_proxy_gap_leading_term_is_half_score_variance():
    """PARK page D.2: for small within-block score deviations the gap between
    the exact log-mass and the centroid estimate is, to leading order, half the
    within-block variance of the scaled scores."""
    rng = np.random.default_rng(3)
    d, b = 64, 32
    q = rng.standard_normal(d)
    center = rng.standard_normal(d)
    dev = rng.standard_normal((b, d))
    ratios = []
    for eps in (1e-1, 1e-2, 1e-3):
        keys = center + eps * dev
        s = R.proxy_logits(q[None, :], keys.mean(0)[None, :], np.array([b]))[0, 0]
        z = torch.from_numpy(keys @ q / math.sqrt(d))
        gap = torch.logsumexp(z, 0).item() - s
        var = z.var(unbiased=False).item()
        ratios.append(gap / (0.5 * var))
    assert abs(ratios[-1] - 1) < 1e-2
    assert abs(ratios[-1] - 1) < abs(ratios[0] - 1)


def test_proxy_is_not_symmetric_in_query_and_key():
    rng = np.random.default_rng(4)
    Qbar, Kbar = rng.standard_normal((5, 8)), rng.standard_normal((5, 8))
    n = np.array([4, 4, 4, 4, 1])
    s = R.proxy_logits(Qbar, Kbar, n)
    assert s[1, 2] == pytest.approx(Qbar[1] @ Kbar[2] / math.sqrt(8) + math.log(4), abs=1e-12)
    assert s[3, 4] == pytest.approx(Qbar[3] @ Kbar[4] / math.sqrt(8), abs=1e-12)


def test_block_softmax_matches_torch_and_shift_invariance():
    rng = np.random.default_rng(5)
    s = rng.standard_normal((7, 11)) * 5
    p = R.block_softmax(s)
    assert np.allclose(p, torch.softmax(torch.from_numpy(s), -1).numpy(), rtol=0, atol=1e-15)
    # PARK page A: a common additive offset does not change the softmax,
    # hence nor the routing.
    p2 = R.block_softmax(s + 123.25)
    r1 = R.route_rows(p, 0.8, 1, 11)
    r2 = R.route_rows(p2, 0.8, 1, 11)
    for a, b_ in zip(r1["kept"], r2["kept"]):
        assert np.array_equal(a, b_)


# ---------------------------------------------------------------- routing --

def brute_force_route(w, tau, kmin, kmax):
    """Smallest set whose mass reaches tau, by exhaustive search over subsets.

    w are exact rational weights.  Among sets of the chosen size, the one of
    largest mass wins, remaining ties go to the lexicographically smallest
    index tuple.  The size is then clamped to [kmin, min(kmax, nb)].
    """
    nb = len(w)
    total = sum(w)
    best_of_size = {}
    for k in range(nb + 1):
        best = None
        for S in itertools.combinations(range(nb), k):
            m = sum((w[j] for j in S), Fraction(0))
            if best is None or m > best[0] or (m == best[0] and S < best[1]):
                best = (m, S)
        best_of_size[k] = best
    if tau >= 1:
        kstar = nb
    else:
        kstar = next(k for k in range(nb + 1) if best_of_size[k][0] / total >= Fraction(tau))
    k = min(max(kstar, kmin), kmax, nb)
    return list(best_of_size[k][1])


@pytest.mark.parametrize("seed", range(6))
def test_routing_matches_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    nb = 9
    # integer weights with deliberate ties; exact as binary fractions
    ints = rng.integers(1, 6, size=nb)
    p = ints / ints.sum()
    wts = [Fraction(int(x)) for x in ints]
    for tau in (0.0, 0.1, 0.33, 0.5, 0.75, 0.9, 0.999, 1.0, 1.5):
        for kmin, kmax in ((1, nb), (3, nb), (1, 4), (2, 2), (1, 100)):
            if tau > 0 and tau < 1:
                # skip thresholds that hit a prefix sum exactly: there the
                # answer depends on the rounding of p and the fractions
                cs = np.cumsum(np.sort(ints)[::-1]) / ints.sum()
                if np.any(np.abs(cs - tau) < 1e-12):
                    continue
            got = R.route_rows(p[None, :], tau, kmin, kmax)["kept"][0].tolist()
            assert got == brute_force_route(wts, tau, kmin, kmax), (tau, kmin, kmax, ints)


def test_routing_random_probabilities_brute_force():
    rng = np.random.default_rng(7)
    for _ in range(20):
        nb = int(rng.integers(2, 10))
        p = R.block_softmax(rng.standard_normal((1, nb)) * 3)[0]
        tau = float(rng.uniform(0.05, 0.98))
        got = R.route_rows(p[None, :], tau, 1, nb)["kept"][0].tolist()
        assert got == brute_force_route([Fraction(x) for x in p], tau, 1, nb)


def test_routing_nested_and_monotone_in_tau():
    rng = np.random.default_rng(8)
    p = R.block_softmax(rng.standard_normal((12, 40)) * 4)
    prev = None
    for tau in np.linspace(0.0, 1.0, 41):
        r = R.route_rows(p, float(tau), 1, 40)
        if prev is not None:
            assert np.all(r["k"] >= prev["k"])
            for a, b_ in zip(prev["kept"], r["kept"]):
                assert set(a.tolist()) <= set(b_.tolist())
        prev = r
    assert np.all(prev["k"] == 40)                                  # tau = 1 keeps all
    assert np.all(R.route_rows(p, 0.0, 3, 40)["k"] == 3)            # tau <= 0 -> kmin
    assert np.all(R.route_rows(p, -1.0, 1, 40)["k"] == 1)
    assert np.all(R.route_rows(p, 0.99, 1, 5)["k"] <= 5)            # kmax clamp


def test_routing_kept_mass_reaches_tau_and_prefix_is_minimal():
    rng = np.random.default_rng(9)
    p = R.block_softmax(rng.standard_normal((30, 25)) * 3)
    tau = 0.83
    r = R.route_rows(p, tau, 1, 25)
    for i in range(30):
        kept = r["kept"][i]
        assert p[i, kept].sum() >= tau
        top = np.sort(p[i])[::-1]
        assert top[: len(kept) - 1].sum() < tau          # one fewer block is not enough


# -------------------------------------------------------------- attention --

def _small_case(seed, N, b, d, const_keys=False):
    rng = np.random.default_rng(seed)
    q = R.decode_bf16(rand_bf16(rng, (N, d), 2.0))
    if const_keys:
        nb = -(-N // b)
        base = rand_bf16(rng, (nb, d), 2.0)
        k = R.decode_bf16(np.repeat(base, b, axis=0)[:N])
    else:
        k = R.decode_bf16(rand_bf16(rng, (N, d), 2.0))
    v = R.decode_bf16(rand_bf16(rng, (N, d)))
    return q, k, v


def _route_head(q, k, b, tau, kmin, kmax):
    n = R.block_sizes(q.shape[0], b)
    Qbar, Kbar = R.block_means(q, b), R.block_means(k, b)
    return R.route_rows(R.block_softmax(R.proxy_logits(Qbar, Kbar, n)), tau, kmin, kmax), n


@pytest.mark.parametrize("N,b,d", [(200, 32, 16), (256, 64, 64), (130, 64, 128)])
@pytest.mark.parametrize("residual", [0, 1])
def test_tau_one_is_dense_softmax_attention(N, b, d, residual):
    q, k, v = _small_case(11, N, b, d)
    r, n = _route_head(q, k, b, 1.0, 1, 10 ** 6)
    assert all(len(x) == len(n) for x in r["kept"])
    out = R.attention(q, k, v, r["kept"], b, bool(residual), R.block_means(k, b), R.block_means(v, b))
    assert np.max(np.abs(out - sdpa64(q, k, v))) < 1e-10


@pytest.mark.parametrize("tau", [0.3, 0.7, 0.9])
def test_no_residual_equals_masked_token_matrix(tau):
    """residual = 0: each token attends to exactly the tokens of its kept
    blocks -- checked against library attention with an explicit N x N mask."""
    N, b, d = 250, 32, 32
    q, k, v = _small_case(12, N, b, d)
    r, n = _route_head(q, k, b, tau, 1, 100)
    assert min(r["k"]) < len(n)           # something is actually dropped
    mask = np.zeros((N, N), dtype=bool)
    for i, kept in enumerate(r["kept"]):
        for j in kept:
            mask[i * b: i * b + n[i], j * b: j * b + n[j]] = True
    out = R.attention(q, k, v, r["kept"], b, False)
    assert np.max(np.abs(out - sdpa64(q, k, v, mask))) < 1e-10


@pytest.mark.parametrize("tau", [0.2, 0.6, 0.95])
def test_residual_exact_for_constant_key_blocks(tau):
    """With equal keys inside every block a dropped block's pseudo-key
    reproduces its exact contribution n_j e^{q.k/sqrt d} Vbar_j, so the
    routed output equals dense attention for any tau and any values."""
    N, b, d = 224, 32, 64
    q, k, v = _small_case(13, N, b, d, const_keys=True)
    r, n = _route_head(q, k, b, tau, 1, 100)
    assert min(r["k"]) < len(n)
    out = R.attention(q, k, v, r["kept"], b, True, R.block_means(k, b), R.block_means(v, b))
    assert np.max(np.abs(out - sdpa64(q, k, v))) < 1e-10
    # and dropping the pseudo-keys does change the answer
    out0 = R.attention(q, k, v, r["kept"], b, False)
    assert np.max(np.abs(out0 - sdpa64(q, k, v))) > 1e-3


def test_residual_uses_each_token_query_not_block_mean():
    """Constant keys, varying queries: exactness needs the per-token q."""
    N, b, d = 128, 32, 32
    q, k, v = _small_case(14, N, b, d, const_keys=True)
    r, n = _route_head(q, k, b, 0.5, 1, 4)
    out = R.attention(q, k, v, r["kept"], b, True, R.block_means(k, b), R.block_means(v, b))
    assert np.max(np.abs(out - sdpa64(q, k, v))) < 1e-10


def test_attention_flop_count_dense_closed_form():
    n = R.block_sizes(1000, 64)
    kept = [list(range(len(n)))] * len(n)
    exact, res = R.attention_flops(kept, n, True, 128)
    assert exact == 4 * 1000 * 1000 * 128 and res == 0


# ------------------------------------------------------------ permutation --

def test_gather_scatter_definition_and_round_trip():
    rng = np.random.default_rng(15)
    perm = rng.permutation(37)
    X = np.arange(37, dtype=np.float64)[:, None] * np.ones((1, 3))
    Xp = R.gather_tokens(X, perm)
    assert np.array_equal(Xp[:, 0], perm)                  # Xp[n] = X[perm[n]]
    assert np.array_equal(R.scatter_tokens(Xp, perm), X)


def test_permutation_equivariance_at_tau_one():
    w = get_config("tiny", H=1)
    Q, K, V = make_qkv(w)
    perm = oracle.hilbert_perm(w.grid)
    a = R.forward(Q, K, V, w.b, 1.0, 1, w.nb, 1)
    bb = R.forward(Q, K, V, w.b, 1.0, 1, w.nb, 1, perm=perm)
    assert np.max(np.abs(a["O"] - bb["O"])) < 1e-10


def test_forward_rows_subset_matches_full():
    w = get_config("tiny", H=1)
    Q, K, V = make_qkv(w)
    perm = oracle.hilbert_perm(w.grid)
    full = R.forward(Q, K, V, w.b, 0.8, 1, w.nb, 1, perm=perm)
    rows = np.array([0, 5, 63, 64, 700, 1023])
    part = R.forward(Q, K, V, w.b, 0.8, 1, w.nb, 1, perm=perm, rows={(0, 0): rows})
    # equal up to the BLAS summation order of a different row count
    assert np.max(np.abs(part["O"][(0, 0)] - full["O"][0, 0, rows])) < 1e-13


# ---------------------------------------------------------------- Hilbert --

def test_hilbert_order_one_is_gray_code():
    rows = np.array([[int(x) for x in l.split()] for l in open(os.path.join(GOLDEN, "hilbert_order1.txt"))
                     if l.strip() and not l.startswith("#")])
    coords = rows[:, 1:]
    idx = oracle.hilbert_index(coords, 1)
    assert np.array_equal(idx, rows[:, 0])
    g = np.arange(8) ^ (np.arange(8) >> 1)
    assert np.array_equal(coords[:, 0] * 4 + coords[:, 1] * 2 + coords[:, 2], g)


@pytest.mark.parametrize("bits", [2, 3, 6])
def test_hilbert_is_a_continuous_bijection(bits):
    s = 1 << bits
    t, h, w = np.meshgrid(np.arange(s), np.arange(s), np.arange(s), indexing="ij")
    coords = np.stack([t.ravel(), h.ravel(), w.ravel()], axis=1)
    idx = oracle.hilbert_index(coords, bits)
    assert np.array_equal(np.sort(idx), np.arange(s ** 3))
    walk = coords[np.argsort(idx)]
    steps = np.abs(np.diff(walk, axis=0)).sum(axis=1)
    assert np.all(steps == 1)
    assert np.array_equal(walk[0], [0, 0, 0])


def test_hilbert_perm_on_stress_grid_is_a_bijection_with_local_blocks():
    w = get_config("stress")
    perm = oracle.hilbert_perm(w.grid)
    assert np.array_equal(np.sort(perm), np.arange(w.N))
    T, Hs, W = w.grid
    t, h, ww = np.unravel_index(perm, (T, Hs, W))
    # consecutive tokens in Hilbert order are near each other on the grid
    jumps = np.abs(np.diff(t)) + np.abs(np.diff(h)) + np.abs(np.diff(ww))
    assert np.median(jumps) == 1


# --------------------------------------------------- PAMA block importance --
# PARK page 5.1: each query keeps its own softmax over key blocks; the block's
# importance is the mean of its queries' rows.

def test_pama_hand_computed_two_tokens():
    """d = 4 (sqrt(d) = 2), equal block sizes.  Token 1 has centroid logits
    (ln 3, 0) -> (3/4, 1/4); token 2 has logits (0, 0) -> (1/2, 1/2); PAMA is
    the mean (5/8, 3/8).  The block-mean query instead gives logits
    (ln 3 / 2, 0) -> (sqrt 3, 1) / (sqrt 3 + 1), which differs."""
    l3 = math.log(3.0)
    q = np.array([[2 * l3, 0, 0, 0], [0, 0, 0, 0]], dtype=np.float64)
    Kbar = np.array([[1, 0, 0, 0], [0, 0, 0, 0]], dtype=np.float64)
    n = np.array([128, 128])
    p = R.pama_importance(q, Kbar, n)
    assert np.allclose(p, [5 / 8, 3 / 8], atol=1e-15)
    pc = R.block_softmax(R.proxy_logits(q.mean(axis=0, keepdims=True), Kbar, n))[0]
    s3 = math.sqrt(3.0)
    assert np.allclose(pc, [s3 / (s3 + 1), 1 / (s3 + 1)], atol=1e-15)
    assert abs(p[0] - pc[0]) > 5e-3


def test_pama_block_size_term():
    """Zero centroids: every token's row is n_j / sum n, so a partial block of
    64 against a full one of 128 gets 1/3 (the ln n_j term)."""
    q = np.random.default_rng(0).standard_normal((5, 8))
    p = R.pama_importance(q, np.zeros((2, 8)), np.array([128, 64]))
    assert np.allclose(p, [2 / 3, 1 / 3], atol=1e-15)


def test_pama_equals_centroid_proxy_for_constant_query_blocks():
    """When every token of the query block is the same vector, averaging the
    per-token softmax rows changes nothing: PAMA equals the block-mean proxy
    softmax."""
    rng = np.random.default_rng(3)
    nb, d = 7, 16
    Kbar = rng.standard_normal((nb, d)) * 2
    n = np.array([16] * (nb - 1) + [5])
    q = np.repeat(rng.standard_normal((1, d)) * 3, 16, axis=0)
    p = R.pama_importance(q, Kbar, n)
    pc = R.block_softmax(R.proxy_logits(q[:1], Kbar, n))[0]
    assert np.allclose(p, pc, rtol=0, atol=1e-14)


def test_pama_rows_are_distributions_and_match_torch():
    """Rows are probability vectors; the per-token softmax and the mean agree
    with torch's fp64 softmax and mean on random data."""
    rng = np.random.default_rng(4)
    q = rng.standard_normal((33, 16)) * 4
    Kbar = rng.standard_normal((9, 16))
    n = np.array([64] * 8 + [17])
    p = R.pama_importance(q, Kbar, n)
    assert abs(p.sum() - 1) < 1e-14 and np.all(p >= 0)
    s = torch.from_numpy(q) @ torch.from_numpy(Kbar).T / 4.0 + torch.log(torch.from_numpy(n).double())
    want = torch.softmax(s, dim=-1).mean(dim=0).numpy()
    assert np.allclose(p, want, atol=1e-15)


def test_forward_pama_routes_from_token_rows():
    """forward(routing='pama') feeds route_rows the PAMA rows of each query
    block (checked against a direct evaluation), and at tau = 1 the output is
    the same dense attention as with the centroid routing."""
    w = get_config("tiny", H=1)
    Q, K, V = make_qkv(w)
    ref = R.forward(Q, K, V, w.b, w.tau, w.kmin, w.kmax, w.residual, routing="pama",
                    want_output=False)
    q = R.decode_bf16(Q[0, 0])
    n = R.block_sizes(w.N, w.b)
    Kbar = ref["Kbar"][0, 0]
    for i in (0, 5, w.nb - 1):
        p = R.pama_importance(q[i * w.b:i * w.b + n[i]], Kbar, n)
        assert np.allclose(ref["route"][(0, 0)]["p"][i], p, atol=1e-15)
    a = R.forward(Q, K, V, w.b, 1.0, 1, w.nb, 1, routing="pama")["O"]
    c = R.forward(Q, K, V, w.b, 1.0, 1, w.nb, 1)["O"]
    assert np.allclose(a, c, atol=1e-12)


# ------------------------------------------------- threshold selection (f3) --

def test_threshold_hand_worked_row():
    p = np.array([[0.4, 0.1, 0.3, 0.1, 0.1]])
    cases = [  # (theta, kmin, kmax) -> kept
        ((0.1, 1, 5), [0, 1, 2, 3, 4]),     # >= is inclusive
        ((0.2, 1, 5), [0, 2]),
        ((0.35, 1, 5), [0]),
        ((0.5, 1, 5), [0]),                 # nothing passes: kmin
        ((0.5, 2, 5), [0, 2]),
        ((0.5, 3, 5), [0, 1, 2]),           # three-way tie at 0.1: the lowest index
        ((0.2, 1, 1), [0]),                 # kmax binds
        ((0.0, 1, 9), [0, 1, 2, 3, 4]),     # kmax > nb
    ]
    for (theta, kmin, kmax), want in cases:
        r = R.route_threshold(p, theta, kmin, kmax)
        assert r["kept"][0].tolist() == want, (theta, kmin, kmax)
        assert r["k"][0] == len(want)


def _dyadic_rows(rng, nq, nb, bits=20):
    """Rows of distinct positive dyadic probabilities summing to exactly 1, so
    that every partial sum is exact in fp64."""
    rows = []
    while len(rows) < nq:
        w = rng.integers(1, 1 << 12, nb)
        w[-1] = 0
        w[-1] = (1 << bits) - w.sum()
        if w[-1] > 0 and len(set(w.tolist())) == nb:
            rows.append(w / float(1 << bits))
    return np.array(rows)


def test_threshold_set_is_the_top_p_set_of_its_own_mass():
    """With no clamp binding, the critical set {p >= theta} is exactly what
    the Top-p rule keeps for tau = the mass of that set (a second,
    independent selection routine reaching the same blocks)."""
    rng = np.random.default_rng(21)
    p = _dyadic_rows(rng, 40, 24)
    for theta in (0.01, 0.03, 0.05, 0.08):
        thr = R.route_threshold(p, theta, 1, 24)
        for i in range(len(p)):
            crit = np.nonzero(p[i] >= theta)[0]
            if len(crit) == 0 or len(crit) == 24:
                continue
            tau = float(p[i][crit].sum())
            top = R.route_rows(p[i:i + 1], tau, 1, 24)
            assert np.array_equal(thr["kept"][i], crit)
            assert np.array_equal(top["kept"][0], crit), (theta, i)


def test_threshold_clamped_budget_is_the_heaviest_subset():
    """When a clamp binds, the kept set is the k-subset of largest mass
    (brute force over all subsets; distinct p make it unique)."""
    rng = np.random.default_rng(22)
    p = _dyadic_rows(rng, 12, 8)
    for theta, kmin, kmax in ((0.9, 3, 8), (0.0, 1, 4), (0.2, 5, 6), (0.01, 2, 2)):
        r = R.route_threshold(p, theta, kmin, kmax)
        for i in range(len(p)):
            k = min(max(int(np.count_nonzero(p[i] >= theta)), kmin), kmax, 8)
            best = max(itertools.combinations(range(8), k), key=lambda c: p[i][list(c)].sum())
            assert r["kept"][i].tolist() == list(best)


def test_threshold_sets_are_nested_in_theta():
    rng = np.random.default_rng(23)
    p = R.block_softmax(rng.standard_normal((30, 40)) * 2.0)
    prev = None
    for theta in (0.0, 0.005, 0.01, 0.02, 0.05, 0.1, 0.3, 1.1):
        r = R.route_threshold(p, theta, 2, 30)
        if prev is not None:
            for a, b in zip(r["kept"], prev["kept"]):
                assert set(a.tolist()) <= set(b.tolist())
        prev = r
    assert all(len(k) == 2 for k in prev["kept"])          # theta > 1: kmin


def test_forward_threshold_zero_is_dense_and_rejects_unknown_selection():
    w = get_config("tiny", H=1, grid=(1, 4, 64))
    Q, K, V = make_qkv(w)
    res = R.forward(Q, K, V, w.b, 0.0, 1, w.nb, 1, selection="threshold")
    q, k, v = (R.decode_bf16(X[0, 0]) for X in (Q, K, V))
    np.testing.assert_allclose(res["O"][0, 0], sdpa64(q, k, v), rtol=0, atol=1e-10)
    with pytest.raises(ValueError):
        R.forward(Q, K, V, w.b, 0.5, 1, w.nb, 1, selection="top_k")
