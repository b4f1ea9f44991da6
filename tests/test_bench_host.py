"""Host-side logic of bench.py that needs no GPU: the FLOP count behind the
headline metric, checked against the oracle's definition."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))



@pytest.mark.parametrize("name,ov", [("tiny", {}), ("medium", {"H": 3}), ("wan", {"H": 2}),
                                     ("tiny", {"residual": 0, "grid": (1, 5, 100), "b": 64})])
def test_bench_flop_count_matches_oracle_definition(name, ov):
    """The bench's vectorised FLOP count from a CSR equals the oracle's
    per-row count (4 d per exact query-key pair and per query-pseudo-key
    pair) on random kept sets, including the partial last block."""
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    from oracle import spattn_ref as R
    from workloads import get_config
    w = get_config(name, **ov)
    nb = w.nb
    n = R.block_sizes(w.N, w.b)
    rng = np.random.default_rng(7)
    kept, rp, ci = {}, [0], []
    for bi in range(w.B):
        for hi in range(w.H):
            rows = []
            for i in range(nb):
                k = int(rng.integers(1, nb + 1))
                ks = np.sort(rng.choice(nb, size=k, replace=False))
                if i == 0:
                    ks = np.unique(np.append(ks, nb - 1))      # the partial block at least once
                rows.append(ks)
                ci.extend(ks.tolist())
                rp.append(rp[-1] + len(ks))
            kept[(bi, hi)] = rows
    ex, rs = bench.attention_flops(np.asarray(rp), np.asarray(ci), w, nb)
    want_ex = want_rs = 0
    for key, rows in kept.items():
        e, r = R.attention_flops(rows, n, bool(w.residual), w.d)
        want_ex += e
        want_rs += r
    assert (ex, rs) == (want_ex, want_rs)


def test_attention_recall_extremes_and_a_hand_case():
    """Recall is 1 when every block is kept, and for a hand-built case it is
    the softmax mass of the kept block: two blocks of two tokens, one query
    whose logits are (ln 3, ln 3, 0, 0) (d = 1), kept = {0}: 6/8."""
    sys.path.insert(0, ROOT)
    import math
    import numpy as np
    import torch
    import bench
    B, H, N, d, b = 1, 1, 4, 1, 2
    q = torch.full((B, H, N, d), math.log(3.0), dtype=torch.float64)
    k = torch.tensor([1.0, 1.0, 0.0, 0.0], dtype=torch.float64).view(B, H, N, d)
    rp_all = np.array([0, 2, 4]); ci_all = np.array([0, 1, 0, 1])
    assert bench.attention_recall(q, k, rp_all, ci_all, b, 2, rows_per_head=4) == 1.0
    rp = np.array([0, 1, 2]); ci = np.array([0, 0])
    r = bench.attention_recall(q, k, rp, ci, b, 2, rows_per_head=4)
    assert abs(r - 0.75) < 1e-6


@pytest.mark.parametrize("extra", [[], ["--selection", "threshold", "--theta", "0.05"], ["--routing", "pama"]])
def test_reference_arm_prints_one_contract_line(extra):
    """`bench.py --impl reference` (the oracle on the host cores) prints one
    JSON line with the keys the benchmark contract names, on the tiny
    workload with a short sample."""
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "1", "--warmup", "3", *extra],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e", "impl"):
        assert key in line, key
    assert line["impl"] == "reference" and line["steps"] == 1 and line["warmup"] == 3
    assert line["value"] > 0 and line["higher_is_better"] is True
    assert line["config"]["workload"] == "tiny"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    if extra:
        assert line["config"][extra[0].lstrip("-")] == extra[1]


def test_warmup_below_three_is_refused():
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "1", "--warmup", "2"],
                       capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert r.returncode != 0 and "warmup" in (r.stderr + r.stdout)


def test_reference_arm_on_a_nonzero_rank_prints_nothing():
    """Under torchrun the reference arm runs on rank 0 alone: another rank
    exits 0 without work or output."""
    import subprocess
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--workload", "tiny", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=120, cwd=ROOT, env=env)
    assert r.returncode == 0 and not [l for l in r.stdout.splitlines() if l.startswith("{")]


def test_default_arguments_are_one_gpu_and_a_short_run():
    sys.path.insert(0, ROOT)
    import bench
    a = bench.parse_args([])
    # the headline: the largest configuration that fits one GPU
    assert a.gpus == 1 and a.impl == "ours" and a.workload == "hunyuan"
    assert a.warmup >= 3 and 1 <= a.steps <= 100
    assert a.selection == "top_p" and a.routing == "centroid"


def test_block_override_keeps_the_budget_share():
    """--block 64 doubles the block count of a layer and scales the budget cap with it, so
    the cap keeps the same share of the blocks (never above nb)."""
    sys.path.insert(0, ROOT)
    import bench
    for name in ("medium", "wan", "hunyuan", "stress"):
        base = bench.workload_from_args(bench.parse_args(["--workload", name]))
        w = bench.workload_from_args(bench.parse_args(["--workload", name, "--block", "64"]))
        nb0, nb1 = -(-base.N // base.b), -(-w.N // 64)
        assert w.b == 64 and w.N == base.N and w.tau == base.tau
        assert w.kmax == min(nb1, -(-base.kmax * nb1 // nb0))
    assert bench.workload_from_args(bench.parse_args(["--block", "128"])).b == 128
