"""Multi-rank host logic of bench.py, on CPU with the gloo backend (world
size 2): each rank runs an independent replica (its own seed), timings are
combined as the max over ranks and work as the sum, and the job throughput
is all ranks' work over the slowest rank's time.  The GPU path uses the same
helpers over NCCL; nothing here needs a GPU."""
import os
import socket
import sys
from datetime import timedelta

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        args = bench.parse_args(["--workload", "medium", "--gpus", str(world)])
        w = bench.workload_from_args(args, rank)
        # rank r: step 1+r ms, attention 10-r ms, 100(r+1) FLOPs of work
        maxes, sums = bench.combine_over_ranks([1.0 + rank, 10.0 - rank], [100.0 * (rank + 1)], "cpu")
        q.put((rank, maxes, sums, w.seed, w.name))
    except Exception as e:  # report instead of hanging the parent
        q.put((rank, "error", repr(e), None, None))
    finally:
        dist.destroy_process_group()


def test_combine_over_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, maxes, sums, seed, name in res:
        assert maxes != "error", sums
        assert maxes == [2.0, 10.0]            # max over ranks
        assert sums == [300.0]                 # sum over ranks
        assert name == "medium"
    seeds = [r[3] for r in res]
    assert seeds[1] == seeds[0] + 1000         # independent replicas


def test_single_process_is_pass_through_and_throughput():
    sys.path.insert(0, ROOT)
    import bench
    maxes, sums = bench.combine_over_ranks([3.5, 1.25], [42.0], "cpu")
    assert maxes == [3.5, 1.25] and sums == [42.0]
    # 2e12 FLOPs in 1 ms is 2000 TFLOP/s
    assert bench.job_throughput(2e12, 1.0) == pytest.approx(2000.0)

