"""Pins for the seeded input generator (no attention arithmetic lives there):
its bf16 rounding against torch, the grid positions, the per-head random
streams, and the logit structure the recipe implies.  With W_f ~ N(0, 8^2),
u ~ U(0, 2 pi) and phi = sqrt(2/d) cos(W_f p + u), E[phi(p) . phi(p')] =
exp(-32 |p - p'|^2); with Q = K = a phi + noise and a^2 = 10 sqrt(d), the
expected logit q . k / sqrt(d) is 10 exp(-32 |dp|^2) (40 exp(...) when a is
doubled)."""
import numpy as np
import pytest
import torch

from workloads import (bf16_bits_to_f32, f32_to_bf16_bits, get_config, grid_positions,
                       make_qkv, probe_rows)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(200000).astype(np.float32) * 10.0 ** rng.integers(-6, 6, 200000),
                        # exact ties between two bf16 values: round to even
                        (np.arange(1, 2001, dtype=np.uint32) << 16 | 0x8000).view(np.float32)])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(f32_to_bf16_bits(x), want)
    assert np.array_equal(bf16_bits_to_f32(want), torch.from_numpy(want.view(np.int16)).view(torch.bfloat16).float().numpy())


def test_grid_positions_are_row_major_in_the_unit_cube():
    pos = grid_positions((3, 1, 5))
    assert pos.shape == (15, 3)
    assert np.array_equal(pos[0], [0, 0, 0]) and np.array_equal(pos[-1], [1, 0, 1])
    assert np.array_equal(pos[1], [0, 0, 0.25])            # w varies fastest
    assert np.array_equal(pos[5], [0.5, 0, 0])              # then h (size 1), then t
    assert np.all(pos[:, 1] == 0)                           # a size-1 axis sits at 0


def test_heads_are_independent_streams():
    """Head (b, h) draws from its own stream: the same bytes whatever the
    number of heads or threads."""
    w = get_config("tiny", B=2, H=3)
    Q, K, V = make_qkv(w)
    Q1, K1, V1 = make_qkv(w.with_(B=2, H=2), threads=1)
    for X, Y in ((Q, Q1), (K, K1), (V, V1)):
        assert np.array_equal(X[:, :2], Y)
    assert not np.array_equal(Q[0, 0], Q[0, 1]) and not np.array_equal(Q[0, 0], Q[1, 0])


@pytest.mark.parametrize("name,scale", [("medium", 10.0), ("stress", 40.0)])
def test_logits_follow_the_recipe(name, scale):
    w = get_config(name, B=1, H=4)
    Q, K, V = make_qkv(w)
    pos = grid_positions(w.grid)
    rng = np.random.default_rng(1)
    i = rng.integers(0, w.N, 40000)
    j = np.where(rng.random(40000) < 0.5, i, rng.integers(0, w.N, 40000))   # half on the diagonal
    dist2 = ((pos[i] - pos[j]) ** 2).sum(axis=1)
    for h in range(w.H):
        q = bf16_bits_to_f32(Q[0, h]).astype(np.float64)
        k = bf16_bits_to_f32(K[0, h]).astype(np.float64)
        v = bf16_bits_to_f32(V[0, h]).astype(np.float64)
        s = (q[i] * k[j]).sum(axis=1) / np.sqrt(w.d)
        for lo, hi in ((0.0, 1e-12), (0.005, 0.015), (0.02, 0.04), (0.2, 3.0)):
            m = (dist2 >= lo) & (dist2 <= hi)
            want = scale * np.mean(np.exp(-32.0 * dist2[m]))
            # the feature average over d = 128 frequencies fluctuates by a few percent
            assert abs(s[m].mean() - want) < 0.08 * scale, (h, lo, s[m].mean(), want)
        assert abs(v.mean()) < 0.01 and abs(v.var() - 1.0) < 0.01
        assert abs((q - k).var() - 2 * 0.3 ** 2) < 0.01                  # independent N(0, 0.3^2) noise


@pytest.mark.parametrize("per_block", [1, 3, 64])
def test_probe_rows_are_stratified_over_blocks(per_block):
    for N, b in ((10, 4), (64, 64), (65, 64), (1000, 64), (7, 8)):
        rows = probe_rows(N, b, 3, per_block)
        n = np.array([min(b, N - i * b) for i in range(-(-N // b))])
        assert np.array_equal(np.bincount(rows // b, minlength=len(n)), np.minimum(n, per_block))
        assert np.all(np.diff(rows) > 0) and rows[-1] < N
        assert np.array_equal(rows, probe_rows(N, b, 3, per_block))
