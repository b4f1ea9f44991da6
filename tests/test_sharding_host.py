"""Sequence-sharded callers (block_sparse_attention_33_b200.sharding) on CPU
with the gloo backend: the all-to-all from token shards to head shards and
back moves every element to the right place, and the sharded path around the
oracle (standing in for the kernels, which run per head) equals the
unsharded oracle output on every rank's token shard."""
import os
import socket
import sys
from datetime import timedelta

import numpy as np
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
    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        from block_sparse_attention_33_b200 import sharding as S
        # data movement: a tensor whose entries name their own coordinates
        B, H, N, d = 2, 4 * world, 6 * world, 3
        full = torch.arange(B * H * N * d, dtype=torch.float64).reshape(B, H, N, d)
        n, h = N // world, H // world
        mine = full[:, :, rank * n:(rank + 1) * n].contiguous()
        heads = S.seq_to_head(mine)
        ok_a = torch.equal(heads, full[:, rank * h:(rank + 1) * h])
        ok_b = torch.equal(S.head_to_seq(heads), mine)
        # the path around the oracle on the local heads
        from oracle import spattn_ref as R
        from workloads import bf16_bits_to_f32, f32_to_bf16_bits, get_config, make_qkv
        w = get_config("tiny", H=2 * world, grid=(1, 8, 64), kmax=4, tau=0.8)
        Q, K, V = make_qkv(w)
        ref = R.forward(Q, K, V, w.b, w.tau, w.kmin, w.kmax, w.residual)["O"]
        n = w.N // world
        to_t = lambda X: torch.from_numpy(bf16_bits_to_f32(X[:, :, rank * n:(rank + 1) * n]).astype(np.float64))

        def oracle_heads(qh, kh, vh):
            bits = [f32_to_bf16_bits(x.numpy().astype(np.float32)) for x in (qh, kh, vh)]
            return torch.from_numpy(R.forward(*bits, w.b, w.tau, w.kmin, w.kmax, w.residual)["O"])

        out = S.forward_seq_sharded(to_t(Q), to_t(K), to_t(V), oracle_heads)
        ok_c = np.array_equal(out.numpy(), ref[:, :, rank * n:(rank + 1) * n])
        try:
            S.seq_to_head(torch.zeros(1, world + 1, 2, 1, dtype=torch.float64))
            ok_d = False
        except ValueError:
            ok_d = True
        q.put((rank, ok_a, ok_b, ok_c, ok_d))
    except Exception as e:  # report instead of hanging the parent
        q.put((rank, "error", repr(e), None, None))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_sequence_sharded_path_matches_unsharded(world):
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    for r in sorted(res):
        assert r[1:] == (True, True, True, True), r
