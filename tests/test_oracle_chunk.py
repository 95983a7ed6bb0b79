"""Pins of the oracle's chunk attention (oracle.attention.chunk_decode): the queries of a
just-appended chunk attend causally over the cache ("WUSH-KV: KV Cache Quantization with
Data-Adaptive Transforms", §4.4: a new chunk is appended in full precision and serves its
own attention output before it is quantized).

Each pin checks it against something other than itself: a dense brute force with an
explicit position mask and scipy's softmax, the decode of the newest token, the causal
limit by perturbation (a position past a query's own must not move it, its own must), and
the exact shift of the output when every value moves by a constant."""
import numpy as np
import pytest
from scipy.special import softmax

from oracle import attention, cache as ocache


def _cache(rng, B=2, H=2, n_prefill=300, chunk=6, sink=4, keep=32, flush=16, store=np.float16):
    oc = ocache.Cache(B, H, 128, 2, 1.0, 99.0, sink, keep, flush, capacity=1024, chunk_max=chunk,
                      store_dtype=store)
    T = np.stack([np.linalg.qr(rng.standard_normal((128, 128)))[0] * rng.uniform(0.5, 2.0, 128)
                  for _ in range(H)]).astype(np.float16)

    def tok(n):
        x = rng.standard_normal((B, n, H, 128))
        x[..., [3, 70]] *= 12
        return x.astype(np.float16)

    oc.append(tok(n_prefill), tok(n_prefill), T)   # bulk: quantized on arrival
    oc.append(tok(chunk), tok(chunk), T)           # the chunk: fp16, not yet flushed
    return oc, T


def _brute(oc, q, T, scale):
    """Dense [n, S] logits, -inf above each query's own position, scipy softmax, P @ V."""
    B, n, Hq, d = q.shape
    g = Hq // oc.H
    out = np.zeros(q.shape)
    for b in range(B):
        S = int(oc.S[b])
        allowed = np.arange(S)[None, :] <= (S - n + np.arange(n))[:, None]  # [n, S]
        for h in range(oc.H):
            K, V = oc.keys_hat(b, h), oc.values_hat(b, h)
            Tinv = np.linalg.solve(T[h].astype(np.float64), np.eye(128))   # T^{-1}
            for j in range(h * g, (h + 1) * g):
                qc = q[b, :, j].astype(np.float64) @ Tinv                  # rows of (T^{-T} q)^T
                logits = scale * qc @ K.T
                logits[~allowed] = -np.inf
                out[b, :, j] = softmax(logits, axis=-1) @ V
    return out


@pytest.mark.parametrize("chunk,g", [(6, 4), (1, 2), (16, 1)])
def test_chunk_matches_masked_brute_force(chunk, g):
    rng = np.random.default_rng(chunk * 10 + g)
    oc, T = _cache(rng, chunk=chunk)
    q = rng.standard_normal((2, chunk, 2 * g, 128)).astype(np.float16)
    got = attention.chunk_decode(oc, q, T, 0.088)
    np.testing.assert_allclose(got, _brute(oc, q, T, 0.088), rtol=0, atol=1e-11)


def test_last_chunk_token_is_the_decode_query():
    rng = np.random.default_rng(5)
    oc, T = _cache(rng, chunk=5)
    q = rng.standard_normal((2, 5, 8, 128)).astype(np.float16)
    got = attention.chunk_decode(oc, q, T, 0.1)
    dec = attention.decode(oc, q[:, -1], T, 0.1)
    np.testing.assert_allclose(got[:, -1], dec, rtol=0, atol=1e-12)


def test_causal_limit_by_perturbation():
    """Query t sees its own position S - n + t and nothing after it."""
    rng = np.random.default_rng(6)
    n = 6
    oc, T = _cache(rng, chunk=n)
    q = rng.standard_normal((2, n, 4, 128)).astype(np.float16)
    base = attention.chunk_decode(oc, q, T, 0.1)
    S = int(oc.S[0])
    for t in range(n - 1):
        own, nxt = S - n + t, S - n + t + 1
        saved = oc.v_store[0, 1, nxt].copy()
        oc.v_store[0, 1, nxt] += np.float16(4.0)
        moved = attention.chunk_decode(oc, q, T, 0.1)
        oc.v_store[0, 1, nxt] = saved
        np.testing.assert_array_equal(moved[0, t], base[0, t])       # the next position is hidden
        assert np.abs(moved[0, t + 1, 2:] - base[0, t + 1, 2:]).max() > 1e-6   # ... from t only
        saved = oc.v_store[0, 1, own].copy()
        oc.v_store[0, 1, own] += np.float16(4.0)
        moved = attention.chunk_decode(oc, q, T, 0.1)
        oc.v_store[0, 1, own] = saved
        assert np.abs(moved[0, t, 2:] - base[0, t, 2:]).max() > 1e-6  # its own position is seen
        np.testing.assert_array_equal(moved[0, t, :2], base[0, t, :2])  # other KV head untouched


def test_value_shift_moves_outputs_by_the_shift():
    """Softmax weights sum to one: adding c to every value adds c to every output (a cache
    held in float64 inside the windows, so the shift is exact)."""
    rng = np.random.default_rng(7)
    oc, T = _cache(rng, n_prefill=20, chunk=4, store=np.float64)
    assert not oc.is_quantized(0).any()
    q = rng.standard_normal((2, 4, 4, 128)).astype(np.float16)
    base = attention.chunk_decode(oc, q, T, 0.1)
    oc.v_store += 0.75
    shifted = attention.chunk_decode(oc, q, T, 0.1)
    np.testing.assert_allclose(shifted - base, 0.75, rtol=0, atol=1e-12)
