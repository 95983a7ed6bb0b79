"""Pins of the oracle's RMS-scaled symmetric (QuEST-style) quantizer (oracle/quest.py):
the Gaussian-optimal clipping endpoints and errors of the uniform grid (the classical
optimum uniform quantizer of a unit Gaussian), a Monte Carlo check of the error integral,
the fixed-order fp32 RMS against double precision, power-of-two scaling, the all-zero
group, and nearest-level codes by brute force."""
import numpy as np
import pytest

from oracle import quest as oqt


@pytest.mark.parametrize("bits,step,mse", [(2, 0.9957, 0.1188), (3, 0.5860, 0.03744), (4, 0.3352, 0.01154)])
def test_gaussian_optimal_alpha_matches_the_classical_uniform_quantizer(bits, step, mse):
    """Optimum uniform quantizers of N(0,1) with 2^b levels: spacing and mean squared error
    (the classical table values, 4 significant digits)."""
    a = oqt.gaussian_optimal_alpha(bits)
    assert 2 * a / (2 ** bits - 1) == pytest.approx(step, abs=6e-4)
    assert oqt.grid_mse(a, bits) == pytest.approx(mse, rel=2e-3)
    # a neighbour of the optimum is worse on both sides
    assert oqt.grid_mse(a * 1.02, bits) > oqt.grid_mse(a, bits) < oqt.grid_mse(a * 0.98, bits)


def test_grid_mse_monte_carlo():
    rng = np.random.default_rng(0)
    zeta = rng.standard_normal(2_000_000)
    for bits, alpha in [(2, 1.4), (4, 2.7)]:
        levels = np.linspace(-alpha, alpha, 2 ** bits)
        q = levels[np.argmin(np.abs(np.clip(zeta, -alpha, alpha)[:, None] - levels[None, :]), axis=1)]
        assert np.mean((zeta - q) ** 2) == pytest.approx(oqt.grid_mse(alpha, bits), rel=1e-2)


def test_rms_fp32_is_within_an_ulp_of_double():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((200, 128)) * rng.uniform(0.01, 100, (200, 1))).astype(np.float16)
    got = oqt.rms_fp32(x).astype(np.float64)
    ref = np.sqrt(np.mean(x.astype(np.float64) ** 2, axis=-1))
    assert np.all(np.abs(got - ref) <= 2 * np.spacing(ref.astype(np.float32)).astype(np.float64))


def test_power_of_two_scaling_and_zero_group():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((50, 128)).astype(np.float16)
    a = oqt.gaussian_optimal_alpha(2)
    c0, s0, z0 = oqt.quantize(x, 2, a)
    for k in (1, 2, 4):
        c, s, z = oqt.quantize((x.astype(np.float32) * 2 ** k).astype(np.float16), 2, a)
        np.testing.assert_array_equal(c, c0)
        np.testing.assert_array_equal(s.astype(np.float32), s0.astype(np.float32) * 2 ** k)
        np.testing.assert_array_equal(z.astype(np.float32), z0.astype(np.float32) * 2 ** k)
    c, s, z = oqt.quantize(np.zeros((1, 128), np.float16), 2, a)
    assert s[0] == 0 and z[0] == 0 and not c.any()


@pytest.mark.parametrize("bits", [2, 4])
def test_codes_are_nearest_levels(bits):
    rng = np.random.default_rng(3 + bits)
    x = (rng.standard_normal((100, 128)) * 3).astype(np.float16)
    a = oqt.gaussian_optimal_alpha(bits)
    c, s, z = oqt.quantize(x, bits, a)
    levels = z.astype(np.float64)[:, None] + s.astype(np.float64)[:, None] * np.arange(2 ** bits)[None, :]
    dist = np.abs(x.astype(np.float64)[:, :, None] - levels[:, None, :])
    best = dist.min(axis=-1)
    got = np.take_along_axis(dist, c[..., None].astype(np.int64), axis=-1)[..., 0]
    assert np.all(got <= best + 1e-6 * np.abs(s.astype(np.float64))[:, None])


def _rms_golden():
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "rms_sigma.txt")
    rows = []
    for line in open(path):
        line = line.split("#")[0].split()
        if line:
            sig = [int(t, 16) for t in line[:5]]
            x = np.array([int(t, 16) for t in line[5:]], dtype=np.uint16).view(np.float16)
            rows.append((sig, x))
    return rows


def test_rms_fp32_summation_order_matches_golden_bits():
    """sigma in the declared fixed order, bit for bit, against tests/golden/rms_sigma.txt
    (written by a pure-Python binary32 routine, make_rms_golden.py).  On every stored vector
    that order gives a different fp32 sigma from a plain left-to-right sum and from three
    other groupings, so the pin fixes the order, not just the value to an ulp."""
    rows = _rms_golden()
    assert len(rows) >= 8
    xs = np.stack([x for _, x in rows])
    got = oqt.rms_fp32(xs).astype(np.float32).view(np.uint32)
    for (sig, _), g in zip(rows, got):
        assert int(g) == sig[0], (hex(int(g)), hex(sig[0]))
        assert all(sig[0] != other for other in sig[1:])
