#!/usr/bin/env python
"""Benchmark of routed block-sparse attention (forward) on B200.

One step = the whole hot path on one synthetic attention call: (optional
Hilbert gather +) block-mean pooling, proxy scoring + Top-p routing + CSR,
routed attention with residual pseudo-keys, output (scatter).  Inputs are
resident in HBM when the timed region starts; the L2 is flushed (a 256 MiB
write) between timed steps, outside the timed events.

value = FLOPs actually computed by the attention (4 d per exact query-key
pair plus 4 d per query-pseudo-key pair) / device time of the whole step.
The line also carries the dense-equivalent rate, the fraction of the
measured bf16 tensor peak, and the speedup over the same library's dense
(tau = 1) path on the same inputs.

  python bench.py [--gpus N --steps K --warmup W] [--workload hunyuan]
  python bench.py --impl reference ...   # the fp64 CPU oracle on host cores
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "block-sparse attn fwd: effective TFLOP/s, % of B200 BF16 peak, speedup vs dense"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNELS_PER_STEP = 4  # pool, route, scan, attend (the compact CSR is not asked for)
L2_NOTE = "flushed (256 MiB write between timed steps)"

# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one
# ncu capture of the bench command for that workload, keyed by kernel and
# (workload, heads, tau, residual).  Valid only while the kernel's sources are
# the ones captured: each entry carries a hash of them, and the bench reports
# null when the hash no longer matches.  The HunyuanVideo-like entries (24
# heads) are 3 x the capture of the same layer with 8 heads: the heads are
# independent and every head's key and value tiles are read the same way, so
# the bytes grow with the head count.
MEASURED_TRAFFIC = {
    "attention": {"sources": ["attn_tc.cu", "tc.cuh", "common.cuh", "select.cuh"],
                  "sha": "857b37df0d5c2d2f",
                  "bytes": {("hunyuan", 24, 0.95, 1): 3 * 2727366144}},
    # wan / hunyuan: pool_kernel (contiguous blocks); stress: pool_gather_kernel
    "pool": {"sources": ["pool.cu", "tc.cuh", "common.cuh"],
             "sha": "da762629b964bc69",
             "bytes": {("wan", 8, 0.9, 1): 206850048, ("stress", 8, 0.7, 1): 357913344,
                       ("hunyuan", 24, 0.95, 1): 3 * 746453248}},
}


def measured_traffic(kernel, w, selection="top_p"):
    import hashlib
    ent = MEASURED_TRAFFIC[kernel]
    m = hashlib.sha256()
    try:
        for f in ent["sources"]:
            with open(os.path.join(ROOT, "block_sparse_attention_33_b200", "csrc", f), "rb") as fh:
                m.update(fh.read())
    except OSError:
        return None
    if m.hexdigest()[:16] != ent["sha"]:
        return None
    if kernel == "attention" and selection != "top_p":
        return None   # captured with Top-p selection: other kept sets, other traffic
    return ent["bytes"].get((w.name, w.H, round(w.tau, 6), int(w.residual)))


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="hunyuan",
                    choices=["tiny", "medium", "wan", "hunyuan", "stress"])
    ap.add_argument("--tau", type=float, default=None)
    ap.add_argument("--residual", type=int, default=None)
    ap.add_argument("--routing", choices=["centroid", "pama"], default="centroid",
                    help="block-importance estimate: block-mean centroids, or per-query "
                         "attention-mass aggregation (PAMA)")
    ap.add_argument("--selection", choices=["top_p", "threshold"], default="top_p",
                    help="Top-p on the cumulative mass (tau), or a per-block threshold on p "
                         "(Sol-Attn on-the-fly thresholding; the knob is --theta)")
    ap.add_argument("--inline", action="store_true",
                    help="select inside the attention kernel (SPATTN_SELECT_INLINE): the step is "
                         "pooling + attention, with the same kept blocks")
    ap.add_argument("--theta", type=float, default=0.01,
                    help="per-block probability threshold with --selection threshold")
    ap.add_argument("--no-probe", action="store_true",
                    help="skip the extra timing of the probe-fitted residual correction")
    ap.add_argument("--no-threshold", action="store_true",
                    help="skip the extra timing of threshold selection at --theta")
    ap.add_argument("--heads", type=int, default=None,
                    help="override the number of heads (smaller profiling captures)")
    ap.add_argument("--block", type=int, default=None, choices=[64, 128],
                    help="override the block size b (64-token blocks: two query blocks per "
                         "128-row tile of the attention)")
    ap.add_argument("--no-dense", action="store_true", help="skip the tau = 1 comparison run")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-chunk", type=int, default=0,
                    help="heads per chunk of spattn_forward_host in the e2e figure (host "
                         "tensors, copies overlapped over chunks); 0: the binding's default")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the compact timing of every seeded configuration")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="CPU time budget of the oracle baseline sample")
    return ap.parse_args(argv)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def workload_from_args(args, rank=0):
    from workloads import get_config
    ov = {}
    if args.tau is not None:
        ov["tau"] = args.tau
    if args.selection == "threshold":
        if args.tau is not None:
            raise SystemExit("--selection threshold takes its knob from --theta, not --tau")
        ov["tau"] = args.theta   # the plan's tau argument carries theta
    if args.residual is not None:
        ov["residual"] = args.residual
    if args.heads is not None:
        ov["H"] = args.heads
    if args.block is not None:
        ov["b"] = args.block
        # the budget cap is a block count: keep it the same share of the blocks
        base = get_config(args.workload)
        nb_base = -(-base.N // base.b)
        nb_new = -(-base.N // args.block)
        ov["kmax"] = max(1, min(nb_new, -(-base.kmax * nb_new // nb_base)))
    w = get_config(args.workload, **ov)
    if rank:
        w = w.with_(seed=w.seed + 1000 * rank)   # independent replica per rank
    return w


def combine_over_ranks(maxes, sums, device):
    """Every rank's timings (max over ranks: the job ends with its slowest
    replica) and work (summed over ranks).  One all-reduce per kind, the same
    on every rank; returns (maxes, sums) as lists of floats."""
    import torch
    import torch.distributed as dist
    out_max, out_sum = list(maxes), list(sums)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if maxes:
            t = torch.tensor(maxes, dtype=torch.float64, device=device)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            out_max = t.tolist()
        if sums:
            t = torch.tensor(sums, dtype=torch.float64, device=device)
            dist.all_reduce(t, op=dist.ReduceOp.SUM)
            out_sum = t.tolist()
    return out_max, out_sum


def job_throughput(total_flops, step_ms):
    """Whole-job TFLOP/s: all ranks' FLOPs over the slowest rank's step time."""
    return total_flops / (step_ms * 1e-3) / 1e12


def attention_recall(q, k, row_ptr, col_idx, b, nb, perm=None, rows_per_head=64, seed=0):
    """Attention recall of the kept mask (PARK page 3.2: the share of the
    full attention weight that the kept blocks cover), averaged over a
    seeded sample of query tokens per head.  q, k: [B, H, N, d] torch
    tensors (any device); row_ptr/col_idx: the CSR (numpy); perm: the
    token permutation (gather) or None.  Dense softmax in fp32 on the
    sampled rows only."""
    import torch
    B, H, N, d = q.shape
    rng = np.random.default_rng(seed)
    total, count = 0.0, 0
    for bi in range(B):
        for hi in range(H):
            qp, kp = q[bi, hi], k[bi, hi]
            if perm is not None:
                pi = torch.as_tensor(np.asarray(perm, dtype=np.int64), device=q.device)
                qp, kp = qp[pi], kp[pi]
            sel = np.sort(rng.choice(N, size=min(rows_per_head, N), replace=False))
            logits = (qp[torch.as_tensor(sel, device=q.device)].float() @ kp.float().T) / float(d) ** 0.5
            w = torch.softmax(logits, dim=-1).cpu().numpy()          # [rows, N]
            blk = np.arange(N) // b
            for ri, tok in enumerate(sel):
                row = (bi * H + hi) * nb + tok // b
                kept = col_idx[row_ptr[row]:row_ptr[row + 1]]
                mask = np.isin(blk, kept)
                total += float(w[ri, mask].sum())
                count += 1
    return total / max(count, 1)


def attention_flops(row_ptr, col_idx, w, nb):
    """(exact, residual) FLOPs: 4 d per query-key pair, from the CSR."""
    b, N, d = w.b, w.N, w.d
    n_last = N - (nb - 1) * b
    rows = len(row_ptr) - 1
    k = np.diff(row_ptr).astype(np.int64)
    row_id = np.repeat(np.arange(rows), k)
    has_last = np.bincount(row_id[col_idx[: row_ptr[-1]] == nb - 1], minlength=rows)
    keys_per_row = b * k - (b - n_last) * has_last
    n_i = np.full(rows, b, np.int64)
    n_i[np.arange(rows) % nb == nb - 1] = n_last
    exact = 4 * d * int(np.sum(n_i * keys_per_row))
    res = 4 * d * int(np.sum(n_i * (nb - k))) if w.residual else 0
    return exact, res


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [x.get("num_threads", 1) for x in threadpool_info() if x.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_sample(w, seconds, Q=None, K=None, V=None, perm=None, routing="centroid",
                  selection="top_p"):
    """Time the fp64 oracle on a bounded sample of the workload.

    Sample: head (0, 0) -- decode, gather, block means, proxy, routing of all
    its query blocks -- then routed attention of successive query blocks of
    that head until `seconds` of wall time have passed.  Returns
    (TFLOP/s of the sampled attention, description).
    """
    from oracle import spattn_ref as R
    from workloads import make_qkv
    if Q is None:
        Q, K, V = make_qkv(w.with_(H=1, B=1))
    t0 = time.perf_counter()
    q = R.gather_tokens(R.decode_bf16(Q[0, 0]), perm)
    k = R.gather_tokens(R.decode_bf16(K[0, 0]), perm)
    v = R.gather_tokens(R.decode_bf16(V[0, 0]), perm)
    n = R.block_sizes(w.N, w.b)
    Qb, Kb, Vb = R.block_means(q, w.b), R.block_means(k, w.b), R.block_means(v, w.b)
    if routing == "pama":
        starts = np.concatenate([[0], np.cumsum(n)[:-1]])
        p = np.stack([R.pama_importance(q[s0:s0 + nj], Kb, n) for s0, nj in zip(starts, n)])
    else:
        p = R.block_softmax(R.proxy_logits(Qb, Kb, n))
    select = R.route_threshold if selection == "threshold" else R.route_rows
    route = select(p, w.tau, w.kmin, w.kmax)
    flops = 0
    blocks = 0
    order = np.random.default_rng(0).permutation(len(n))
    for i in order:
        rows = np.arange(i * w.b, i * w.b + n[i])
        R.attention(q, k, v, route["kept"], w.b, bool(w.residual), Kb, Vb, rows=rows)
        nk = int(n[route["kept"][i]].sum())
        flops += 4 * w.d * int(n[i]) * (nk + (len(n) - len(route["kept"][i]) if w.residual else 0))
        blocks += 1
        if time.perf_counter() - t0 > seconds:
            break
    dt = time.perf_counter() - t0
    desc = (f"head 0 of {w.name}: pooling + routing of all {len(n)} query blocks, then routed "
            f"attention of {blocks} random query blocks ({blocks * w.b} query tokens); "
            f"{dt:.1f} s wall; TFLOP/s = sampled attention FLOPs / total wall time")
    return flops / dt / 1e12, desc, dt


def run_reference(args):
    """The oracle (fp64, CPU) timed on the host cores on the same config."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = workload_from_args(args)
    from workloads import make_qkv
    Q, K, V = make_qkv(w.with_(H=1, B=1))
    perm = None
    if w.hilbert:
        import oracle
        perm = oracle.hilbert_perm(w.grid)
    per_step = max(1.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(w, per_step, Q, K, V, perm, args.routing, args.selection)
    vals, times, desc = [], [], ""
    for _ in range(args.steps):
        v, desc, dt = oracle_sample(w, per_step, Q, K, V, perm, args.routing, args.selection)
        vals.append(v)
        times.append(dt)
    value = float(np.mean(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * float(np.mean(times)), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        # the GPU arm's config, so that the two lines describe the same workload
        "config": dict(config_of(w, L2_NOTE), routing=args.routing, selection=args.selection,
                       inline_selection=bool(args.inline)),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(),
                         "kind": "oracle", "sample": "each step: " + desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_of(w, l2):
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "b": w.b,
            "nb": w.nb, "tau": w.tau, "kmin": w.kmin, "kmax": w.kmax, "residual": w.residual,
            "hilbert": w.hilbert, "grid": list(w.grid), "global_batch": w.B, "seq_len": w.N,
            "parallelism": "replicas", "l2": l2}


# The seeded configurations and the knob values they are quoted at.
PER_CONFIG = (("tiny", {}), ("medium", {}), ("medium", {"residual": 0}),
              ("wan", {"tau": 0.8}), ("wan", {}), ("wan", {"tau": 0.95}),
              ("hunyuan", {"tau": 0.8}), ("hunyuan", {}),
              ("stress", {}), ("stress", {"residual": 0}))


def measure_configs(sp, main_w, main_qkv, main_perm, main_dense_ms, timed, as_graph, graphs,
                    dev, steps):
    """Step time (route + attend, CUDA-graph replays, L2 flushed between
    steps), attention TFLOP/s, kept fraction and speedup over the dense path
    of every entry of PER_CONFIG.  Inputs of the main workload are reused."""
    import torch
    from workloads import get_config, make_qkv
    out = []
    by_name = {}
    for name, ov in PER_CONFIG:
        by_name.setdefault(name, []).append(ov)
    for name, variants in by_name.items():
        base = get_config(name)
        if name == main_w.name and main_w.H == base.H:
            (q, k, v), perm = main_qkv, main_perm
        else:
            Qh, Kh, Vh = make_qkv(base)
            q, k, v = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
                       for x in (Qh, Kh, Vh))
            del Qh, Kh, Vh
            perm = sp.spattn_hilbert_perm(*base.grid) if base.hilbert else None
        o = torch.empty_like(q)
        B, H, N, d = q.shape
        dense_flops = 4 * N * N * d * B * H
        dense_ms = main_dense_ms if (q is main_qkv[0] and main_dense_ms) else None
        if dense_ms is None:
            dplan = sp.Plan(B, H, N, d, base.b, 1.0, 1, 1 << 30, base.residual, perm, device=dev)
            n0 = len(graphs)
            td = timed([as_graph(lambda: dplan.forward(q, k, v, o))], steps, 3)
            dense_ms = float(np.mean([x[0] for x in td]))
            del graphs[n0:]
            dplan.close()
        for ov in variants:
            w = base.with_(**ov)
            plan = sp.Plan(B, H, N, d, w.b, w.tau, w.kmin, w.kmax, w.residual, perm, device=dev)
            try:
                rp = torch.zeros(B * H * plan.nb + 1, dtype=torch.int32, device=dev)
                ci = torch.zeros(max(plan.col_capacity, 1), dtype=torch.int32, device=dev)
                plan.route(q, k, v, rp, ci)
                torch.cuda.synchronize(dev)
                rpn, cin = rp.cpu().numpy(), ci.cpu().numpy()
                exact, resid = attention_flops(rpn, cin, w, plan.nb)
                n0 = len(graphs)
                t = timed([as_graph(lambda: plan.route(q, k, v)),
                           as_graph(lambda: plan.attend(q, k, v, o))], steps, 3)
                del graphs[n0:]
                status = plan.check()
            finally:
                plan.close()
            r_ms = float(np.mean([x[0] for x in t]))
            a_ms = float(np.mean([x[1] for x in t]))
            kept = float(np.diff(rpn).sum()) / (B * H * plan.nb * plan.nb)
            out.append({"workload": name, "tau": w.tau, "residual": w.residual, "H": H, "N": N,
                        "ms_per_step": r_ms + a_ms, "route_ms": r_ms, "attend_ms": a_ms,
                        "step_tflops": (exact + resid) / ((r_ms + a_ms) * 1e-3) / 1e12,
                        "attn_tflops": (exact + resid) / (a_ms * 1e-3) / 1e12,
                        "dense_equiv_tflops": dense_flops / ((r_ms + a_ms) * 1e-3) / 1e12,
                        "kept_fraction": kept, "dense_ms": dense_ms,
                        "speedup_vs_dense": dense_ms / (r_ms + a_ms),
                        "dense_over_computed_flops": dense_flops / max(exact + resid, 1),
                        "status": int(status)})
        del q, k, v, o
        torch.cuda.empty_cache()
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    import block_sparse_attention_33_b200 as sp
    from block_sparse_attention_33_b200 import build
    if rank == 0 and not build.up_to_date():
        build.build()
    if world > 1:
        dist.barrier()
    sp.lib()
    from workloads import make_qkv

    w = workload_from_args(args, rank)
    Qh, Kh, Vh = make_qkv(w)
    perm = sp.spattn_hilbert_perm(*w.grid) if w.hilbert else None
    B, H, N, d = Qh.shape

    def dev_bf16(x):
        return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)

    q, k, v = dev_bf16(Qh), dev_bf16(Kh), dev_bf16(Vh)
    o = torch.empty_like(q)
    routing = sp.ROUTING_PAMA if args.routing == "pama" else sp.ROUTING_CENTROID
    if args.selection == "threshold":
        routing |= sp.SELECT_THRESHOLD
    if args.inline:
        if args.routing == "pama":
            raise SystemExit("--inline selects from the centroid estimate")
        routing |= sp.SELECT_INLINE
    plan = sp.Plan(B, H, N, d, w.b, w.tau, w.kmin, w.kmax, w.residual, perm, device=dev,
                   routing=routing)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def timed(fn_list, steps, warmup):
        """Per step: flush L2, then events around each fn; returns [steps][len(fns)] ms."""
        for _ in range(warmup):
            flush.zero_()
            for fn in fn_list:
                fn()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(fn_list) + 1)]
               for _ in range(steps)]
        for s in range(steps):
            flush.zero_()
            evs[s][0].record(stream)
            for i, fn in enumerate(fn_list):
                fn()
                evs[s][i + 1].record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        return [[evs[s][i].elapsed_time(evs[s][i + 1]) for i in range(len(fn_list))]
                for s in range(steps)]

    # Each timed piece is captured once into a CUDA graph and replayed, so a
    # slow host cannot leave the GPU idle between the timed launches (eager
    # launches are the fallback if capture fails; the line says which).
    launch = {"mode": "cuda_graph"}

    def as_graph(fn):
        try:
            fn()
            torch.cuda.synchronize(dev)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, capture_error_mode="thread_local"):
                fn()
            torch.cuda.synchronize(dev)
            graphs.append(g)
            return g.replay
        except Exception as e:  # pragma: no cover - depends on the driver
            torch.cuda.synchronize(dev)
            launch["mode"] = "eager"
            launch["capture_error"] = repr(e)[:200]
            return fn

    graphs = []
    row_ptr = torch.zeros(B * H * plan.nb + 1, dtype=torch.int32, device=dev)
    col_idx = torch.zeros(max(plan.col_capacity, 1), dtype=torch.int32, device=dev)
    # routing once to count FLOPs (deterministic: same every step)
    plan.route(q, k, v, row_ptr, col_idx)
    torch.cuda.synchronize(dev)
    rp, ci = row_ptr.cpu().numpy(), col_idx.cpu().numpy()
    exact, resid = attention_flops(rp, ci, w, plan.nb)
    step_flops = exact + resid
    kept_frac = float(np.diff(rp).sum()) / (B * H * plan.nb * plan.nb)
    try:   # a diagnostic: never let it stop the measurement
        recall = attention_recall(q, k, rp, ci, w.b, plan.nb, perm,
                                  rows_per_head=max(8, 512 // max(1, B * H)))
    except Exception as e:  # pragma: no cover
        recall = {"error": repr(e)[:200]}
    dense_flops = 4 * N * N * d * B * H

    clocks = ClockSampler(local)
    clocks.start()
    # the step: routing (pooling, proxy, selection, work order) then the
    # attention; with --inline, pooling then the attention, which selects
    # the same blocks itself
    first = (lambda: plan.pool(q, k, v)) if args.inline else (lambda: plan.route(q, k, v))
    t = timed([as_graph(first), as_graph(lambda: plan.attend(q, k, v, o))],
              args.steps, args.warmup)
    clk = clocks.stop()
    route_ms = float(np.mean([x[0] for x in t]))
    attend_ms = float(np.mean([x[1] for x in t]))
    step_ms = route_ms + attend_ms

    status = plan.check()
    if status != 0:
        raise RuntimeError(f"device status {status}: {sp.spattn_last_error()}")

    # max over ranks of the step time (device-timed), work summed over ranks
    (step_ms, attend_ms), (total_flops,) = combine_over_ranks([step_ms, attend_ms],
                                                              [float(step_flops)], dev)
    value = job_throughput(total_flops, step_ms)
    peaks, peak_kind = load_peaks()
    # The attention kernel's peak: the burst figure when the timed region is
    # short, the sustained (power-capped) one when the timed launches keep
    # the GPU busy for a second or more, as the long layers do.
    sustained = attend_ms * args.steps >= 1000.0
    bf16_key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    bf16_peak = float(peaks.get(bf16_key, FALLBACK_PEAKS[bf16_key]))
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    attn_tflops = step_flops / (attend_ms * 1e-3) / 1e12

    # the same library's dense path (tau = 1) on the same inputs
    dense_ms = None
    if not args.no_dense:
        dplan = sp.Plan(B, H, N, d, w.b, 1.0, 1, 1 << 30, w.residual, perm, device=dev)
        n_graphs = len(graphs)
        td = timed([as_graph(lambda: dplan.forward(q, k, v, o))], max(3, args.steps // 3), 2)
        dense_ms = float(np.mean([x[0] for x in td]))
        (dense_ms,), _ = combine_over_ranks([dense_ms], [], dev)
        del graphs[n_graphs:]      # release the dense graph before its plan
        dplan.close()

    # kernel breakdown: the pooling kernel alone (HBM-bound)
    tp = timed([as_graph(lambda: plan.pool(q, k, v))], max(3, args.steps // 3), 2)
    pool_ms = float(np.mean([x[0] for x in tp]))
    # routing (proxy logits, softmax, selection, order): the proxy GEMM's FLOPs
    # on fp32 FMA lanes; its time is the step's route chain minus the pooling
    route_flops = (4.0 * B * H * N * plan.nb * d if args.routing == "pama"     # two passes over every token
                   else 2.0 * B * H * plan.nb * plan.nb * d)
    fp32_peak = 148 * 128 * 2 * float(peaks.get("sm_max_mhz", 1965.0)) * 1e6 / 1e12
    tok_bytes = B * H * N * d * 2
    pool_bytes = 3 * tok_bytes + B * H * plan.nb * d * (3 * 4 + 2 * 2)
    if perm is not None:
        pool_bytes += 3 * tok_bytes

    # end to end through the public call with host buffers
    # routing reuse across calls: pooling of the current inputs (new means for
    # the residual) + attention with the kept lists of the last route
    plan.route(q, k, v)   # the reuse step attends with this routing's lists
    tr = timed([as_graph(lambda: plan.pool(q, k, v)), as_graph(lambda: plan.attend(q, k, v, o))],
               max(3, args.steps // 3), 2)
    reuse_ms = float(np.mean([x[0] + x[1] for x in tr]))
    (reuse_ms,), _ = combine_over_ranks([reuse_ms], [], dev)

    # end to end through the public host-buffer call: spattn_forward_host on
    # pinned host tensors (copies in, the path, the copy out, overlapped over
    # chunks of heads); the plain sequence of torch copies around
    # spattn_forward is kept beside it for comparison
    e2e = e2e_copies = None
    if not args.no_e2e:
        qh, kh, vh = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
                      for x in (Qh, Kh, Vh))
        oh = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
        chunk = args.e2e_chunk if args.e2e_chunk > 0 else sp.default_chunk_heads(B * H)

        def pipe_step():
            plan.forward_host(qh, kh, vh, oh, chunk_heads=chunk)

        def copies_step():
            q.copy_(qh, non_blocking=True)
            k.copy_(kh, non_blocking=True)
            v.copy_(vh, non_blocking=True)
            plan.forward(q, k, v, o)
            oh.copy_(o, non_blocking=True)

        tpp = timed([pipe_step], max(3, args.steps // 3), 3)
        pipe_ms = float(np.mean([x[0] for x in tpp]))
        (pipe_ms,), _ = combine_over_ranks([pipe_ms], [], dev)
        pipe_status = plan.check()
        e2e = {"value": total_flops / (pipe_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "ms_per_step": pipe_ms, "h2d_bytes_per_step": 3 * tok_bytes,
               "d2h_bytes_per_step": tok_bytes, "chunk_heads": chunk,
               "what": "spattn_forward_host through the C ABI: pinned host Q, K, V in, host O "
                       "out, copies overlapped with the path over chunks of heads"}
        if pipe_status != sp.OK:   # reported in the line: every rank still takes the same steps
            e2e["error"] = f"device status {pipe_status}: {sp.spattn_last_error()}"
        te = timed([copies_step], max(3, args.steps // 3), 3)
        copies_ms = float(np.mean([x[0] for x in te]))
        (copies_ms,), _ = combine_over_ranks([copies_ms], [], dev)
        e2e_copies = {"value": total_flops / (copies_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                      "ms_per_step": copies_ms, "h2d_bytes_per_step": 3 * tok_bytes,
                      "d2h_bytes_per_step": tok_bytes,
                      "what": "torch copies in, spattn_forward, torch copy out, one after the "
                              "other"}

    # threshold selection (p >= theta, Sol-Attn on-the-fly thresholding) on the
    # same inputs: a second plan, timed like the main step; one rank only
    thresh = None
    if world == 1 and args.selection == "top_p" and not args.no_threshold:
        try:
            tplan = sp.Plan(B, H, N, d, w.b, args.theta, w.kmin, w.kmax, w.residual, perm,
                            device=dev, routing=routing | sp.SELECT_THRESHOLD)
            trp = torch.zeros(B * H * tplan.nb + 1, dtype=torch.int32, device=dev)
            tci = torch.zeros(max(tplan.col_capacity, 1), dtype=torch.int32, device=dev)
            tplan.route(q, k, v, trp, tci)
            torch.cuda.synchronize(dev)
            t_rp, t_ci = trp.cpu().numpy(), tci.cpu().numpy()
            t_exact, t_resid = attention_flops(t_rp, t_ci, w, tplan.nb)
            n_graphs = len(graphs)
            tt = timed([as_graph(lambda: tplan.route(q, k, v)),
                        as_graph(lambda: tplan.attend(q, k, v, o))], max(3, args.steps // 3), 2)
            t_route = float(np.mean([x[0] for x in tt]))
            t_attend = float(np.mean([x[1] for x in tt]))
            status = tplan.check()
            del graphs[n_graphs:]      # release its graphs before its plan
            tplan.close()
            if status != sp.OK:
                raise RuntimeError(f"device status {status}: {sp.spattn_last_error()}")
            thresh = {"theta": args.theta,
                      "kept_fraction": float(np.diff(t_rp).sum()) / (B * H * tplan.nb * tplan.nb),
                      "ms_per_step": t_route + t_attend, "route_ms": t_route, "attend_ms": t_attend,
                      "value": (t_exact + t_resid) / ((t_route + t_attend) * 1e-3) / 1e12,
                      "attn_tflops": (t_exact + t_resid) / (t_attend * 1e-3) / 1e12,
                      "unit": "TFLOP/s",
                      "what": "per-block threshold p >= theta in the route kernel, same attention"}
            # the same threshold selected inside the attention pass: pooling
            # + attention, no routing launch and no kept lists
            if routing == sp.ROUTING_CENTROID:
                fplan = sp.Plan(B, H, N, d, w.b, args.theta, w.kmin, w.kmax, w.residual, perm,
                                device=dev,
                                routing=routing | sp.SELECT_THRESHOLD | sp.SELECT_INLINE)
                n_graphs = len(graphs)
                tf = timed([as_graph(lambda: fplan.pool(q, k, v)),
                            as_graph(lambda: fplan.attend(q, k, v, o))], max(3, args.steps // 3), 2)
                f_pool = float(np.mean([x[0] for x in tf]))
                f_attend = float(np.mean([x[1] for x in tf]))
                fstatus = fplan.check()
                del graphs[n_graphs:]
                fplan.close()
                thresh["inline"] = {
                    "ms_per_step": f_pool + f_attend, "pool_ms": f_pool, "attend_ms": f_attend,
                    "value": (t_exact + t_resid) / ((f_pool + f_attend) * 1e-3) / 1e12,
                    "unit": "TFLOP/s", "status": int(fstatus),
                    "speedup_vs_route_attend": (t_route + t_attend) / (f_pool + f_attend),
                    "what": "the same threshold selected inside the attention kernel "
                            "(SPATTN_SELECT_INLINE): pooling + attention, no routing launch"}
        except Exception as ex:   # reported in the line; the measurements above stand
            thresh = {"error": f"{type(ex).__name__}: {ex}"[:300], "theta": args.theta}

    # probe-fitted residual correction (SparsePR) of the routed output: enough
    # probe rows per block for at least 2 (d + 1) rows per head; one rank only
    probe = None
    if world == 1 and not args.no_probe:
        try:
            from workloads import probe_rows
            per_block = max(1, -(-2 * (d + 1) // plan.nb))
            pr = np.stack([np.stack([probe_rows(N, w.b, (w.seed, 7, bi, hi), per_block)
                                     for hi in range(H)]) for bi in range(B)]).astype(np.int32)
            M = int(pr.shape[-1])
            pr_dev = torch.from_numpy(pr).to(dev)
            p_lam, p_r = 100.0, 16
            plan.forward(q, k, v, o)
            n_graphs = len(graphs)
            tpc = timed([as_graph(lambda: plan.probe_correct(q, k, v, o, pr_dev, p_lam, p_r))],
                        max(3, args.steps // 3), 2)
            p_ms = float(np.mean([x[0] for x in tpc]))
            del graphs[n_graphs:]
            status = plan.check()
            if status != sp.OK:
                raise RuntimeError(f"device status {status}: {sp.spattn_last_error()}")
            probe = {"ms": p_ms, "share_of_step": p_ms / step_ms, "M": M, "per_block": per_block,
                     "lam": p_lam, "r": p_r,
                     "dense_row_flops": 4.0 * B * H * M * N * d,
                     "what": "probe-fitted residual correction: exact probe rows, ridge fit, "
                             "Jacobi subspace, O += O (B P) + b P"}
        except Exception as ex:   # reported in the line; the measurements above stand
            probe = {"error": f"{type(ex).__name__}: {ex}"[:300]}

    # every seeded configuration (and its knob variants) timed the same way,
    # each beside the same library's dense (tau = 1) path on its inputs; one
    # rank only
    per_config = None
    if world == 1 and not args.no_per_config:
        try:
            per_config = measure_configs(sp, w, (q, k, v), perm, dense_ms, timed, as_graph, graphs,
                                         dev, max(3, min(args.steps, 10)))
        except Exception as ex:   # reported in the line; the measurements above stand
            per_config = {"error": f"{type(ex).__name__}: {ex}"[:300]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        val, desc, _ = oracle_sample(w, args.cpu_seconds, perm=perm, routing=args.routing,
                                     selection=args.selection)
        cpu = {"value": val, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "sample": desc}

    try:
        graphs.clear()
        plan.close()
    except Exception:
        if not any(x and "error" in x for x in (thresh, probe)):
            raise   # a failure already recorded in the line may also fail the clean-up
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": dict(config_of(w, L2_NOTE),
                           routing=args.routing, selection=args.selection,
                           inline_selection=bool(args.inline)),
            "dense_equiv_tflops": dense_flops * world / (step_ms * 1e-3) / 1e12,
            "attn_tflops": attn_tflops,
            "pct_of_bf16_peak": 100.0 * attn_tflops / bf16_peak,
            "speedup_vs_dense": (dense_ms / step_ms) if dense_ms else None,
            "dense_ms_per_step": dense_ms,
            "kept_fraction": kept_frac,
            "attention_recall": recall,
            "flops_exact": exact, "flops_residual": resid,
            "kernels_ms": {"route_total": route_ms, "attend": attend_ms, "pool": pool_ms},
            "reuse_step": {"ms_per_step": reuse_ms,
                           "value": job_throughput(total_flops, reuse_ms), "unit": "TFLOP/s",
                           "what": "pool + attend with the kept lists of the last route"},
            "roofline": {"bound": "tensor", "kernel": "attention", "achieved": attn_tflops,
                         "peak": bf16_peak, "unit": "TFLOP/s", "frac": attn_tflops / bf16_peak,
                         "peak_kind": f"{peak_kind} bf16 dense "
                                      f"({'sustained' if sustained else 'burst'})",
                         "traffic": measured_traffic("attention", w, args.selection), "traffic_unit": "bytes/launch"},
            "roofline_route": {"bound": "alu", "kernel": "route + scan",
                               "achieved": route_flops / (max(route_ms - pool_ms, 1e-6) * 1e-3) / 1e12,
                               "peak": fp32_peak, "unit": "TFLOP/s",
                               "frac": route_flops / (max(route_ms - pool_ms, 1e-6) * 1e-3) / 1e12 / fp32_peak,
                               "peak_kind": "fp32 FMA: 148 SMs x 128 lanes x 2 FLOP x max SM clock",
                               "time_ms": route_ms - pool_ms, "traffic": None},
            "roofline_pool": {"bound": "hbm", "kernel": "pool", "achieved": pool_bytes / (pool_ms * 1e-3) / 1e9,
                              "peak": hbm_peak, "unit": "GB/s",
                              "frac": pool_bytes / (pool_ms * 1e-3) / 1e9 / hbm_peak,
                              "peak_kind": f"{peak_kind} copy bandwidth",
                              "traffic": measured_traffic("pool", w), "traffic_unit": "bytes/launch"},
            "clocks": clk,
            "launch": launch,
            "e2e": e2e,
            "e2e_torch_copies": e2e_copies,
            "per_config": per_config,
            "threshold_selection": thresh,
            "probe_correction": probe,
            # pool, route, scan, attend; pool and attend with --inline
            "gpu_launches": (2 if args.inline else KERNELS_PER_STEP) * args.steps,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
