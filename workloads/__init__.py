"""Seeded synthetic workloads for routed block-sparse attention.

This module only draws random numbers and lays them out; it holds none of the
attention method's arithmetic (no pooling, scoring, routing or softmax).  Both
the CUDA path's tests/benchmark and the fp64 oracle read the bf16 bytes it
produces, so every consumer sees exactly the same inputs.

Input recipe (the pages evaluate on 720p video-DiT latents -- Wan and
HunyuanVideo at 50 denoising steps, PARK page section 6.1 -- which need
trained weights; these synthetic tensors stand in for them):

* latent grid T x Hs x W, original token order n = (t*Hs + h)*W + w;
* position p = (t/(T-1), h/(Hs-1), w/(W-1)), a coordinate is 0 when its
  dimension has size 1;
* per (batch, head): W_f ~ N(0, 8^2)^{d x 3}, u ~ U(0, 2 pi)^d,
  phi(p) = sqrt(2/d) * cos(W_f p + u);
* Q = a*phi + N(0, 0.3^2), K = a*phi + N(0, 0.3^2) (same phi, independent
  noise), V ~ N(0, 1), with a = sqrt(10*sqrt(d)) (doubled for the stress case);
* everything is drawn in float64, rounded to float32, then to bf16 with
  round-to-nearest-even.

The random stream of (batch b, head h) is numpy's PCG64 seeded with
[seed, b, h]; within a head the draws come in the order W_f, u, Q noise,
K noise, V.  Heads are independent streams so they can be drawn in parallel.
"""
from __future__ import annotations

import dataclasses
import math
from concurrent.futures import ThreadPoolExecutor
from typing import Optional

import numpy as np

__all__ = [
    "Workload", "CONFIGS", "get_config", "grid_positions", "make_qkv",
    "f32_to_bf16_bits", "bf16_bits_to_f32", "probe_rows",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic attention call: shapes, routing knobs and generator knobs."""
    name: str
    B: int
    H: int
    d: int
    grid: tuple  # (T, Hs, W)
    b: int
    tau: float
    kmin: int
    kmax: int
    residual: int
    hilbert: bool = False
    a_scale: float = 1.0
    seed: int = 0

    @property
    def N(self) -> int:
        T, Hs, W = self.grid
        return T * Hs * W

    @property
    def nb(self) -> int:
        return -(-self.N // self.b)

    @property
    def amp(self) -> float:
        return math.sqrt(10.0 * math.sqrt(self.d)) * self.a_scale

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five seeded configurations.  Seeds are the configuration index.
CONFIGS = {
    "tiny": Workload("tiny", B=1, H=2, d=64, grid=(4, 16, 16), b=64, tau=0.9,
                     kmin=1, kmax=16, residual=1, seed=0),
    "medium": Workload("medium", B=1, H=8, d=128, grid=(8, 32, 32), b=128, tau=0.9,
                       kmin=1, kmax=64, residual=1, seed=1),
    "wan": Workload("wan", B=1, H=40, d=128, grid=(21, 30, 52), b=128, tau=0.9,
                    kmin=1, kmax=256, residual=1, seed=2),
    "hunyuan": Workload("hunyuan", B=1, H=24, d=128, grid=(33, 45, 80), b=128, tau=0.95,
                        kmin=1, kmax=929, residual=1, seed=3),
    # kmax = 25% of the 256 blocks; amplitude doubled; Hilbert order on
    # the 64^3 cube that encloses the 21x30x52 grid.
    "stress": Workload("stress", B=1, H=40, d=128, grid=(21, 30, 52), b=128, tau=0.7,
                       kmin=1, kmax=64, residual=1, hilbert=True, a_scale=2.0, seed=4),
}


def get_config(name: str, **overrides) -> Workload:
    w = CONFIGS[name]
    return w.with_(**overrides) if overrides else w


def grid_positions(grid) -> np.ndarray:
    """[N, 3] float64 positions in [0,1]^3, row-major (t, h, w) token order."""
    T, Hs, W = grid

    def axis(n):
        return np.arange(n, dtype=np.float64) / (n - 1) if n > 1 else np.zeros(1)

    t, h, w = np.meshgrid(axis(T), axis(Hs), axis(W), indexing="ij")
    return np.stack([t.ravel(), h.ravel(), w.ravel()], axis=1)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns uint16 bits.

    Inputs are finite, so no NaN special case is needed.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def _draw_head(w: Workload, pos: np.ndarray, bi: int, hi: int):
    rng = np.random.default_rng([w.seed, bi, hi])
    d, N = w.d, pos.shape[0]
    W_f = rng.normal(0.0, 8.0, size=(d, 3))
    u = rng.uniform(0.0, 2.0 * math.pi, size=d)
    phi = math.sqrt(2.0 / d) * np.cos(pos @ W_f.T + u)
    q = w.amp * phi + rng.normal(0.0, 0.3, size=(N, d))
    k = w.amp * phi + rng.normal(0.0, 0.3, size=(N, d))
    v = rng.normal(0.0, 1.0, size=(N, d))
    return tuple(f32_to_bf16_bits(x.astype(np.float32)) for x in (q, k, v))


def make_qkv(w: Workload, threads: Optional[int] = None):
    """Return (Q, K, V) as uint16 bf16 bit arrays of shape [B, H, N, d].

    Tokens are in the original row-major grid order; any permutation is
    applied later by whoever consumes them.
    """
    pos = grid_positions(w.grid)
    shape = (w.B, w.H, w.N, w.d)
    Q = np.empty(shape, np.uint16)
    K = np.empty(shape, np.uint16)
    V = np.empty(shape, np.uint16)
    jobs = [(bi, hi) for bi in range(w.B) for hi in range(w.H)]

    def run(job):
        bi, hi = job
        Q[bi, hi], K[bi, hi], V[bi, hi] = _draw_head(w, pos, bi, hi)

    n_threads = threads if threads is not None else min(len(jobs), 16)
    if n_threads <= 1:
        for j in jobs:
            run(j)
    else:
        with ThreadPoolExecutor(n_threads) as ex:
            list(ex.map(run, jobs))
    return Q, K, V


def probe_rows(N: int, b: int, seed, per_block: int = 1) -> np.ndarray:
    """Probe tokens of one head for the probe-fitted residual correction:
    per_block distinct tokens drawn from each block of b tokens (all of a
    block shorter than that), ascending.  seed is anything numpy's
    default_rng accepts."""
    rng = np.random.default_rng(seed)
    nb = (N + b - 1) // b
    out = []
    for i in range(nb):
        n_i = min(b, N - i * b)
        k = min(per_block, n_i)
        out.extend(i * b + np.sort(rng.choice(n_i, k, replace=False)))
    return np.asarray(out, dtype=np.int64)
