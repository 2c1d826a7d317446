"""Pins of the oracle's two-tap dynamic depthwise conv (tamsi page, "L’idée,
sans le papier": a two-tap convolution before/after each attention and MLP;
myaiexp page, "主な機能": 2-tap dynamic convolution).

out_t = x_t + (W_a x_t) * x_t + (W_b x_t) * x_{t-1},  x_{-1} = x_prev,
W_tap = [W_a; W_b] in [2H, H] (row h of W_a = row h, row h of W_b = row H + h).
Pinned by hand-computed integer cases (exact in fp64), the special weights
that reduce it to closed forms, and a 3-cycle permutation that fixes the
orientation of W_tap.
"""
import numpy as np
import pytest

import synth


def test_hand_case_integers(orc):
    # H = 2, T = 3, one sequence.
    x = np.array([[[1, 2], [3, -1], [0, 2]]], np.float32)
    x_prev = np.array([[2, -3]], np.float32)
    W_a = np.array([[1, 0], [1, 1]], np.float32)        # a = (x0, x0 + x1)
    W_b = np.array([[0, 2], [-1, 0]], np.float32)       # b = (2 x1, -x0)
    out = orc.dynconv2(x, x_prev, np.concatenate([W_a, W_b]))
    # t=0: x=(1,2) a=(1,3) b=(4,-1) xp=(2,-3): out=(1+1*1+4*2, 2+3*2+(-1)(-3)) = (10, 11)
    # t=1: x=(3,-1) a=(3,2) b=(-2,-3) xp=(1,2): out=(3+9-2, -1-2-6) = (10, -9)
    # t=2: x=(0,2) a=(0,2) b=(4,0) xp=(3,-1): out=(0+0+12, 2+4+0) = (12, 6)
    np.testing.assert_array_equal(out, [[[10, 11], [10, -9], [12, 6]]])


def _rand(seed, B, T, H):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, T, H)).astype(np.float32),
            rng.standard_normal((B, H)).astype(np.float32))


def test_zero_weights_is_identity(orc):
    x, xp = _rand(1, 2, 4, 8)
    out = orc.dynconv2(x, xp, np.zeros((16, 8), np.float32))
    np.testing.assert_array_equal(out, x.astype(np.float64))


def test_identity_a_tap(orc):
    x, xp = _rand(2, 2, 5, 6)
    w = np.concatenate([np.eye(6), np.zeros((6, 6))]).astype(np.float32)
    out = orc.dynconv2(x, xp, w)
    xd = x.astype(np.float64)
    np.testing.assert_allclose(out, xd + xd * xd, rtol=1e-15, atol=0)


def test_identity_b_tap_uses_previous_token_and_x_prev(orc):
    x, xp = _rand(3, 3, 4, 5)
    w = np.concatenate([np.zeros((5, 5)), np.eye(5)]).astype(np.float32)
    out = orc.dynconv2(x, xp, w)
    xd = x.astype(np.float64)
    prev = np.concatenate([xp.astype(np.float64)[:, None], xd[:, :-1]], axis=1)
    np.testing.assert_allclose(out, xd + xd * prev, rtol=1e-15, atol=0)


def test_orientation_three_cycle(orc):
    """W_a = P with P[h][pi(h)] = 1, pi a 3-cycle: a_t[h] = x_t[pi(h)]; the
    transpose would give x_t[pi^-1(h)], which differs for a 3-cycle."""
    x, xp = _rand(4, 1, 2, 3)
    pi = [1, 2, 0]
    P = np.zeros((3, 3), np.float32)
    P[np.arange(3), pi] = 1
    out = orc.dynconv2(x, xp, np.concatenate([P, np.zeros((3, 3), np.float32)]))
    xd = x.astype(np.float64)
    np.testing.assert_allclose(out, xd + xd[..., pi] * xd, rtol=1e-15, atol=0)


def test_bf16_matches_widened_fp32(orc):
    x, xp = _rand(5, 2, 3, 16)
    rng = np.random.default_rng(6)
    w = (rng.standard_normal((32, 16)) / 4).astype(np.float32)
    bx, bxp, bw = synth.to_bf16_bits(x), synth.to_bf16_bits(xp), synth.to_bf16_bits(w)
    a = orc.dynconv2(bx, bxp, bw)
    b = orc.dynconv2(synth.bf16_bits_to_f32(bx), synth.bf16_bits_to_f32(bxp),
                     synth.bf16_bits_to_f32(bw))
    np.testing.assert_array_equal(a, b)


def test_matches_einsum_on_random_input(orc):
    """Library contraction (numpy einsum) of the same definition on a random case."""
    x, xp = _rand(7, 2, 6, 12)
    rng = np.random.default_rng(8)
    w = rng.standard_normal((24, 12)).astype(np.float32)
    xd, wd = x.astype(np.float64), w.astype(np.float64)
    a = np.einsum("hk,btk->bth", wd[:12], xd)
    b = np.einsum("hk,btk->bth", wd[12:], xd)
    prev = np.concatenate([xp.astype(np.float64)[:, None], xd[:, :-1]], axis=1)
    np.testing.assert_allclose(orc.dynconv2(x, xp, w), xd + a * xd + b * prev, rtol=1e-12,
                               atol=1e-12)
