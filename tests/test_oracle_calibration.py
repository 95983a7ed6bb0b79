"""Pins of the oracle's calibration Gram matrices (oracle/calibration.py).

Each pin holds independently of the oracle's own formula:
  - brute force: pure-Python triple loops on a tiny input;
  - a worked case: one one-hot token gives a single nonzero entry a^2 on the diagonal;
  - invariants: symmetry, positive semidefiniteness, and trace = sum of squared norms;
  - the transform relation: for k' = T k the Gram matrix becomes T M T^T.  T is a
    non-symmetric random matrix, so a transposed operand fails this pin.  For orthogonal
    T the trace is unchanged (the pages' Appendix B: an orthogonal transform leaves both
    traces unchanged);
  - accumulation: the Gram matrix of two batches is the sum of theirs;
  - head independence: one head's data never reaches another head's Gram matrix.
"""
import numpy as np
import scipy.stats

from oracle import calibration as ocal
from oracle import transform as otr


def _keys(rng, n, h, d=128):
    return rng.standard_normal((n, h, d)).astype(np.float16)


def test_gram_matches_brute_force_loops():
    rng = np.random.default_rng(11)
    x = _keys(rng, 3, 2, 16)
    m = ocal.gram(x)
    assert m.shape == (2, 16, 16)
    for h in range(2):
        for i in range(16):
            for j in range(16):
                acc = 0.0
                for t in range(3):
                    acc += float(x[t, h, i]) * float(x[t, h, j])
                assert m[h, i, j] == acc


def test_gram_of_one_hot_token():
    x = np.zeros((1, 1, 128), dtype=np.float16)
    x[0, 0, 41] = -3.5
    m = ocal.gram(x)
    expect = np.zeros((1, 128, 128))
    expect[0, 41, 41] = 12.25
    np.testing.assert_array_equal(m, expect)


def test_gram_symmetric_psd_and_trace():
    rng = np.random.default_rng(12)
    x = _keys(rng, 200, 3)
    m = ocal.gram(x)
    np.testing.assert_array_equal(m, np.transpose(m, (0, 2, 1)))
    for h in range(3):
        assert np.linalg.eigvalsh(m[h]).min() > -1e-9 * np.trace(m[h])
        sq = sum(float(v) ** 2 for v in x[:, h, :].astype(np.float64).ravel())
        np.testing.assert_allclose(np.trace(m[h]), sq, rtol=1e-12)


def test_gram_under_a_key_transform():
    rng = np.random.default_rng(13)
    x = rng.standard_normal((64, 1, 128))
    t = rng.standard_normal((128, 128))  # general, non-symmetric
    m = ocal.gram(x)[0]
    xt = np.einsum("ri,nhi->nhr", t, x)  # k' = T k per token
    np.testing.assert_allclose(ocal.gram(xt)[0], t @ m @ t.T, rtol=1e-9, atol=1e-9 * np.abs(t @ m @ t.T).max())
    q = scipy.stats.ortho_group.rvs(128, random_state=4)
    mq = ocal.gram(np.einsum("ri,nhi->nhr", q, x))[0]
    np.testing.assert_allclose(np.trace(mq), np.trace(m), rtol=1e-12)
    h = otr.hadamard(128)
    mh = ocal.gram(np.einsum("ri,nhi->nhr", h, x))[0]
    np.testing.assert_allclose(np.trace(mh), np.trace(m), rtol=1e-12)


def test_gram_accumulates_over_batches_and_keeps_heads_apart():
    rng = np.random.default_rng(14)
    a = _keys(rng, 50, 2)
    b = _keys(rng, 30, 2)
    np.testing.assert_allclose(ocal.gram(np.concatenate([a, b])), ocal.gram(a) + ocal.gram(b), rtol=1e-12)
    c = a.copy()
    c[:, 1, :] = rng.standard_normal((50, 128)).astype(np.float16)
    np.testing.assert_array_equal(ocal.gram(c)[0], ocal.gram(a)[0])
    assert not np.array_equal(ocal.gram(c)[1], ocal.gram(a)[1])
