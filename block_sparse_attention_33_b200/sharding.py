"""Sequence-sharded callers: re-shard tokens to heads and back around the path.

Every (batch, head) pair is an independent attention call through pooling,
routing and attention, so the path itself needs no exchange when each rank
holds whole heads.  A caller whose activations are split along the sequence
(rank j holding tokens [j*N/W, (j+1)*N/W) of every head) needs one
all-to-all before the path (sequence shards -> head shards) and one after it
(head shards -> sequence shards).  These helpers do exactly that over
torch.distributed (NCCL between GPUs; gloo on the host for tests) and run the
path on the local heads in between.

Layouts are [B, H, N, d] throughout; W = world size must divide H and N.
"""
from __future__ import annotations

from typing import Callable


def _world_size(group) -> int:
    import torch.distributed as dist
    return dist.get_world_size(group)


def seq_to_head(x, group=None):
    """[B, H, N/W, d] (this rank's tokens, every head) -> [B, H/W, N, d] (this
    rank's heads, every token).  Rank j receives heads [j*H/W, (j+1)*H/W);
    tokens come back in sequence order."""
    import torch
    import torch.distributed as dist
    W = _world_size(group)
    B, H, n, d = x.shape
    if H % W:
        raise ValueError(f"the world size {W} must divide the head count {H}")
    h = H // W
    send = x.reshape(B, W, h, n, d).permute(1, 0, 2, 3, 4).contiguous()   # chunk j -> rank j
    recv = torch.empty_like(send)                                          # chunk j <- rank j
    dist.all_to_all_single(recv, send, group=group)
    return recv.permute(1, 2, 0, 3, 4).reshape(B, h, W * n, d)


def head_to_seq(y, group=None):
    """Inverse of seq_to_head: [B, H/W, N, d] -> [B, H, N/W, d]."""
    import torch
    import torch.distributed as dist
    W = _world_size(group)
    B, h, N, d = y.shape
    if N % W:
        raise ValueError(f"the world size {W} must divide the sequence length {N}")
    n = N // W
    send = y.reshape(B, h, W, n, d).permute(2, 0, 1, 3, 4).contiguous()   # chunk j -> rank j
    recv = torch.empty_like(send)                                          # chunk j <- rank j
    dist.all_to_all_single(recv, send, group=group)
    return recv.permute(1, 0, 2, 3, 4).reshape(B, W * h, n, d)


def forward_seq_sharded(q, k, v, forward_heads: Callable, group=None, out=None):
    """Attention of a sequence-sharded caller: q, k, v are this rank's token
    shards [B, H, N/W, d]; forward_heads(qh, kh, vh) -> oh runs the path on
    whole heads [B, H/W, N, d] (for instance a Plan made for B, H/W, N, d);
    returns (or writes into `out`) this rank's token shard of the output."""
    qh, kh, vh = (seq_to_head(x, group) for x in (q, k, v))
    o = head_to_seq(forward_heads(qh, kh, vh), group)
    if out is None:
        return o
    out.copy_(o)
    return out


def plan_forward(plan) -> Callable:
    """forward_heads for forward_seq_sharded from a Plan over the local heads."""
    import torch

    def run(qh, kh, vh):
        o = torch.empty_like(qh)
        plan.forward(qh, kh, vh, o)
        return o
    return run
