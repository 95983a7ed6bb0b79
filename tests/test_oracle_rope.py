"""Pins of the oracle's RMSNorm and RoPE (oracle/rope.py) against what mathematics fixes:
the complex-rotation form of rotate-half RoPE, its relative-position property, norm
preservation and its closed form on a unit vector; RMSNorm's unit RMS, scale invariance
and elementwise gain."""
import math

import numpy as np
import pytest

from oracle import rope as orope


@pytest.mark.parametrize("theta", [1e4, 5e5, 1e6])
def test_rope_equals_complex_rotation(theta):
    """Pair (i, i + d/2) as the complex number x_i + j x_{i+d/2}: RoPE multiplies it by
    exp(j * pos * theta^(-2i/d))."""
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 128))
    pos = np.array([0, 1, 17, 32767, 131071])
    z = x[:, :64] + 1j * x[:, 64:]
    w = np.exp(1j * pos[:, None] * np.power(theta, -np.arange(64) / 64.0))
    ref = z * w
    out = orope.rope(x, pos, theta)
    np.testing.assert_allclose(out[:, :64], ref.real, atol=1e-9)
    np.testing.assert_allclose(out[:, 64:], ref.imag, atol=1e-9)


def test_rope_relative_position_and_norm():
    rng = np.random.default_rng(2)
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    for m, n, delta in [(5, 3, 100), (0, 4096, 7), (131000, 17, 70)]:
        a = orope.rope(q, m, 1e6) @ orope.rope(k, n, 1e6)
        b = orope.rope(q, m + delta, 1e6) @ orope.rope(k, n + delta, 1e6)
        assert abs(a - b) <= 1e-9 * (1 + abs(a))
    for p in (0, 1, 999, 131071):
        r = orope.rope(q, p, 5e5)
        np.testing.assert_allclose(np.hypot(r[:64], r[64:]), np.hypot(q[:64], q[64:]), rtol=1e-12)
    np.testing.assert_array_equal(orope.rope(q, 0, 1e4), q)


def test_rope_unit_vector_closed_form():
    """e_0 rotates at frequency 1 (i = 0): (cos p, ..., sin p at index d/2, ...)."""
    e0 = np.zeros(128)
    e0[0] = 1.0
    for p in (1, 2, 1000):
        out = orope.rope(e0, p, 1e4)
        assert out[0] == pytest.approx(math.cos(p), abs=1e-12)
        assert out[64] == pytest.approx(math.sin(p), abs=1e-12)
        assert np.count_nonzero(np.abs(out) > 1e-15) <= 2


def test_rmsnorm_properties():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 128)) * 7
    y = orope.rmsnorm(x, None, eps=0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-12)
    np.testing.assert_allclose(orope.rmsnorm(3.5 * x, None, 0.0), y, rtol=1e-12)
    g = rng.uniform(0.5, 2, 128)
    np.testing.assert_allclose(orope.rmsnorm(x, g, 1e-6), orope.rmsnorm(x, None, 1e-6) * g, rtol=1e-12)
    # eps keeps a zero vector finite
    assert np.all(orope.rmsnorm(np.zeros(128), None, 1e-6) == 0)


def test_prepare_rounds_once_to_fp16():
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((3, 128)) * 2).astype(np.float16)
    out = orope.prepare(x, np.array([5, 6, 7]), 1e6, gain=None, eps=1e-6, norm=True)
    assert out.dtype == np.float16
    exact = orope.rope(orope.rmsnorm(x.astype(np.float64), None, 1e-6), np.array([5, 6, 7]), 1e6)
    assert np.max(np.abs(out.astype(np.float64) - exact) / np.maximum(np.abs(exact), 2 ** -14)) <= 2 ** -11
