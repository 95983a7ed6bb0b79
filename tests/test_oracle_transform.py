"""Pins of the oracle's normalised Hadamard transform (oracle/transform.py): scipy's
Hadamard matrix, orthonormality and symmetry (so it is its own compensation), norm and
trace preservation, and exact compensation in the attention oracle."""
import numpy as np
import scipy.linalg

from oracle import attention as oatt
from oracle import transform as otr


def test_hadamard_equals_scipy_and_is_orthonormal():
    h = otr.hadamard(128)
    np.testing.assert_array_equal(h * np.sqrt(128), scipy.linalg.hadamard(128).astype(np.float64))
    np.testing.assert_allclose(h @ h.T, np.eye(128), atol=1e-13)
    np.testing.assert_array_equal(h, h.T)
    np.testing.assert_allclose(oatt.compensation(h[None])[0], h, atol=1e-13)


def test_hadamard_preserves_norm_and_gram_trace():
    rng = np.random.default_rng(5)
    k = rng.standard_normal((64, 128))
    h = otr.hadamard(128)
    kp = k @ h.T
    np.testing.assert_allclose(np.linalg.norm(kp, axis=1), np.linalg.norm(k, axis=1), rtol=1e-12)
    assert np.trace(kp.T @ kp) == np.float64(np.trace(kp.T @ kp))
    np.testing.assert_allclose(np.trace(kp.T @ kp), np.trace(k.T @ k), rtol=1e-12)


def test_hadamard_flattens_an_outlier_channel():
    """A single large channel spreads evenly over all 128 dimensions (the reason a
    Hadamard rotation helps a per-token quantizer)."""
    x = np.zeros(128)
    x[37] = 10.0
    y = otr.hadamard(128) @ x
    np.testing.assert_allclose(np.abs(y), 10.0 / np.sqrt(128), rtol=1e-12)
