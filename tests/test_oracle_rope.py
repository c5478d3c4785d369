"""Pins of oracle/rope.py: hand-computed rotations, the relative-position property, and
the special cases (position 0, pass-through past rope_dim)."""

from __future__ import annotations

import math

import numpy as np
import pytest

from oracle import rope as R

COS1, SIN1 = 0.5403023058681398, 0.8414709848078965          # cos(1), sin(1)
COS01, SIN01 = 0.9999500004166653, 0.009999833334166664      # cos(0.01), sin(0.01)


def test_hand_rotation_interleaved():
    # d = rope_dim = 4, base 10000: pair 0 turns by p rad, pair 1 by p * 10000^(-1/2) = 0.01 p
    out = R.rope_rows(np.array([[1.0, 0.0, 0.0, 1.0]]), np.array([1]), 4)
    np.testing.assert_allclose(out[0], [COS1, SIN1, -SIN01, COS01], rtol=0, atol=1e-15)


def test_hand_rotation_half_split():
    # pairs (0, 2) and (1, 3)
    out = R.rope_rows(np.array([[1.0, 0.0, 0.0, 1.0]]), np.array([1]), 4, interleaved=False)
    np.testing.assert_allclose(out[0], [COS1, -SIN01, SIN1, COS01], rtol=0, atol=1e-15)


def test_position_zero_and_pass_through():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((3, 8))
    np.testing.assert_array_equal(R.rope_rows(x, np.zeros(3, int), 8), x)
    out = R.rope_rows(x, np.array([5, 6, 7]), 4)              # only the first 4 values turn
    np.testing.assert_array_equal(out[:, 4:], x[:, 4:])
    assert not np.allclose(out[:, :4], x[:, :4])


@pytest.mark.parametrize("interleaved", [True, False])
def test_relative_position_and_norms(interleaved):
    # <R(p) q, R(s) k> depends on p - s only; rotations keep every pair's norm
    rng = np.random.default_rng(1)
    q, k = rng.standard_normal((1, 16)), rng.standard_normal((1, 16))
    dots = []
    for p, s in [(10, 3), (107, 100), (7, 0)]:
        a = R.rope_rows(q, np.array([p]), 16, interleaved=interleaved)
        b = R.rope_rows(k, np.array([s]), 16, interleaved=interleaved)
        dots.append((a @ b.T).item())
        np.testing.assert_allclose(np.linalg.norm(a), np.linalg.norm(q), rtol=1e-14)
    np.testing.assert_allclose(dots, dots[0], rtol=1e-12)
    assert not math.isclose(dots[0], (q @ k.T).item(), rel_tol=1e-6)


def test_heads_share_the_token_angle():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((2, 3, 8))
    out = R.rope_heads(q, np.array([4, 9]), 8)
    for t, p in enumerate([4, 9]):
        for h in range(3):
            np.testing.assert_array_equal(out[t, h], R.rope_rows(q[t, h][None], np.array([p]), 8)[0])
