"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: numbers the
pages print, closed forms, library routines (numpy.percentile, scipy softmax,
numpy.linalg.solve), brute force on tiny inputs, or invariants the pages state.
No test here needs a GPU.
"""
import os

import numpy as np
import pytest
from scipy.special import softmax

from oracle import attention, cache as ocache, footprint, quantizer

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- footprint
def _golden_rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                yield line


def test_footprint_matches_printed_figures():
    """cnshai.top "kv-cache-quantization-fp8-training", "The KV cache is the wall"."""
    rows = list(_golden_rows("footprint.txt"))
    assert len(rows) == 5
    for row in rows:
        name, n_layer, n_kv, d, seq, bits, value = row.split()
        n_layer, n_kv, d, seq, bits, value = map(int, (n_layer, n_kv, d, seq, bits, value))
        if name == "values_per_token":
            got = footprint.values_per_token(n_layer, n_kv, d)
        elif bits == 16:
            got = footprint.bytes_fp16(n_layer, n_kv, d, seq)
        else:
            got = footprint.bytes_codes(n_layer, n_kv, d, seq, bits)
        assert got == value, name
    # the post's "8x" and "4x" reductions
    assert footprint.bytes_fp16(32, 32, 128, 131072) == 8 * footprint.bytes_codes(32, 32, 128, 131072, 2)
    assert footprint.bytes_fp16(32, 32, 128, 131072) == 4 * footprint.bytes_codes(32, 32, 128, 131072, 4)


# ---------------------------------------------------------------- percentile
@pytest.mark.parametrize("p,expect", [(1.0, 1.27), (99.0, 125.73), (0.5, 0.635), (99.5, 126.365),
                                      (0.0, 0.0), (100.0, 127.0), (50.0, 63.5)])
def test_percentile_closed_form_on_ramp(p, expect):
    """x_j = j: the p-th percentile is p/100 * 127 exactly (up to fp32 rounding)."""
    x = np.arange(128, dtype=np.float16)[None, :]
    lo, _ = quantizer.clip_range(x, p, 100.0)
    assert abs(float(lo[0]) - expect) <= 2 * np.spacing(np.float32(expect))


def test_percentile_matches_numpy_linear_method():
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((500, 128)) * rng.uniform(0.1, 30, (500, 1))).astype(np.float16)
    x[:, 7] *= 20
    for p_lo, p_hi in ((1.0, 99.0), (0.5, 99.5), (10.0, 90.0), (0.0, 100.0)):
        lo, hi = quantizer.clip_range(x, p_lo, p_hi)
        ref_lo = np.percentile(x.astype(np.float64), p_lo, axis=-1, method="linear")
        ref_hi = np.percentile(x.astype(np.float64), p_hi, axis=-1, method="linear")
        tol = 4e-7 * np.maximum(np.abs(ref_lo), np.abs(ref_hi)).max() + 1e-30
        np.testing.assert_allclose(lo, ref_lo, rtol=0, atol=tol * 10)
        np.testing.assert_allclose(hi, ref_hi, rtol=0, atol=tol * 10)


# ---------------------------------------------------------------- quantizer
@pytest.mark.parametrize("bits", [2, 4])
def test_codes_are_nearest_level_bruteforce(bits):
    """Every code is the nearest of the 2^b levels z + s c (clamped), by brute force."""
    rng = np.random.default_rng(5 + bits)
    x = (rng.standard_normal((400, 128)) * 3).astype(np.float16)
    x[:, 3] *= 20
    c, s, z = quantizer.quantize(x, bits, 1.0, 99.0)
    assert c.dtype == np.uint8 and c.min() >= 0 and c.max() <= 2 ** bits - 1
    levels = z.astype(np.float64)[:, None, None] + s.astype(np.float64)[:, None, None] * np.arange(2 ** bits)
    dist = np.abs(x.astype(np.float64)[:, :, None] - levels)
    best = dist.argmin(-1)
    # exclude elements within fp32 rounding of a midpoint between two levels
    u = (x.astype(np.float64) - z.astype(np.float64)[:, None]) / s.astype(np.float64)[:, None]
    near_tie = np.abs(u - np.floor(u) - 0.5) < 1e-5
    ok = (best == c) | near_tie
    assert ok.all()
    assert near_tie.mean() < 1e-3
    # below lo -> 0, above hi -> max
    assert (c[x.astype(np.float64) < z.astype(np.float64)[:, None] - 0.5 * s.astype(np.float64)[:, None]] == 0).all()


@pytest.mark.parametrize("bits", [2, 4])
def test_on_grid_vectors_recover_codes(bits):
    """x = z + s c with s a power of two and z fp16: codes come back exactly, step = (hi-lo)/(2^b-1)."""
    rng = np.random.default_rng(21 + bits)
    for _ in range(50):
        s = np.float16(2.0 ** rng.integers(-6, 3))
        z = np.float16(rng.integers(-64, 64) * 0.25)
        c = rng.integers(0, 2 ** bits, 128)
        c[:3] = 0                       # at least 3 copies of each extreme, so both
        c[3:6] = 2 ** bits - 1          # percentiles land on the extremes
        x = (np.float64(z) + np.float64(s) * c).astype(np.float16)
        assert np.array_equal(x.astype(np.float64), np.float64(z) + np.float64(s) * c)
        cq, sq, zq = quantizer.quantize(x[None], bits, 1.0, 99.0)
        assert sq[0] == s and zq[0] == z
        assert np.array_equal(cq[0], c)


@pytest.mark.parametrize("bits", [2, 4])
def test_requantize_dequantized_roundtrip(bits):
    """quant(dequant(c; s, z); s, z) == c (identity transform)."""
    rng = np.random.default_rng(31 + bits)
    x = (rng.standard_normal((300, 128)) * 2).astype(np.float16)
    c, s, z = quantizer.quantize(x, bits, 1.0, 99.0)
    xh = quantizer.dequantize(c, s, z).astype(np.float16)
    c2 = quantizer.quantize_codes(xh, s, z, bits)
    assert np.array_equal(c, c2)


@pytest.mark.parametrize("bits", [2, 4])
def test_power_of_two_scaling_invariance(bits):
    rng = np.random.default_rng(41 + bits)
    x = (rng.standard_normal((200, 128)) * 2).astype(np.float16)
    c, s, z = quantizer.quantize(x, bits, 0.5, 99.5)
    for k in (1, 2, 4):   # stays clear of fp16 subnormals and overflow
        xk = (x.astype(np.float64) * 2.0 ** k).astype(np.float16)
        assert np.array_equal(xk.astype(np.float64), x.astype(np.float64) * 2.0 ** k)
        ck, sk, zk = quantizer.quantize(xk, bits, 0.5, 99.5)
        assert np.array_equal(ck, c)
        assert np.array_equal(sk.astype(np.float64), s.astype(np.float64) * 2.0 ** k)
        assert np.array_equal(zk.astype(np.float64), z.astype(np.float64) * 2.0 ** k)


def test_degenerate_groups():
    x = np.full((1, 128), 1.5, dtype=np.float16)
    c, s, z = quantizer.quantize(x, 2, 1.0, 99.0)
    assert s[0] == 0 and z[0] == np.float16(1.5) and not c.any()
    assert np.array_equal(quantizer.dequantize(c, s, z), x.astype(np.float64))
    # two outliers inside the clipped tails: range collapses, outliers clip to z
    y = np.zeros((1, 128), dtype=np.float16)
    y[0, 5], y[0, 9] = 100, -100
    c, s, z = quantizer.quantize(y, 2, 1.0, 99.0)
    assert s[0] == 0 and z[0] == 0 and not c.any()


# ---------------------------------------------------------------- packing
@pytest.mark.parametrize("bits", [2, 4])
def test_pack_matches_golden_and_roundtrips(bits):
    for row in _golden_rows("pack.txt"):
        b, codes, packed = (t.strip() for t in row.split("|"))
        if int(b) != bits:
            continue
        codes = np.array([int(v) for v in codes.split()], dtype=np.uint8)
        want = np.array([int(v, 16) for v in packed.split()], dtype=np.uint8)
        assert np.array_equal(quantizer.pack(codes, bits), want)
        assert np.array_equal(quantizer.unpack(want, bits), codes)
    rng = np.random.default_rng(bits)
    c = rng.integers(0, 2 ** bits, (64, 128)).astype(np.uint8)
    p = quantizer.pack(c, bits)
    assert p.shape == (64, 128 * bits // 8)
    assert np.array_equal(quantizer.unpack(p, bits), c)


# ---------------------------------------------------------------- Algorithm 2
@pytest.mark.parametrize("sink,keep,flush,chunk_max", [(4, 32, 16, 1), (0, 8, 1, 1), (2, 5, 7, 3),
                                                       (16, 128, 16, 16), (4, 0, 4, 1)])
def test_window_accounting(sink, keep, flush, chunk_max):
    """Invariants §4.4 states: sink + keep full-precision entries persist once the windows
    separate, fewer than S_flush more linger, the quantized region grows in S_flush steps
    and never reaches the recent window; quantized entries never change."""
    rng = np.random.default_rng(sink * 100 + keep * 10 + flush)
    d = 128
    c = ocache.Cache(1, 1, d, 2, 1.0, 99.0, sink, keep, flush, capacity=2000, chunk_max=chunk_max)
    T = np.eye(d, dtype=np.float16)[None]
    frozen = {}
    S = 0
    while S < 1600:
        n = int(rng.choice([1, 1, 1, 2, 3, 9, 17, 40]))
        k = rng.standard_normal((1, n, 1, d)).astype(np.float16)
        v = rng.standard_normal((1, n, 1, d)).astype(np.float16)
        c.append(k, v, T)
        S += n
        Sq = int(c.S_quant[0])
        assert int(c.S[0]) == S
        if Sq:
            assert Sq >= sink + flush and (Sq - sink) % flush == 0
            assert S - Sq >= keep
        fp16_nonsink = S - max(Sq, sink) if S > sink else 0
        slack = n if n <= chunk_max else 0     # a small chunk waits for the next call's flush
        if S >= sink + keep:
            pending = fp16_nonsink - keep
            assert 0 <= pending < flush + slack
        # quantized entries are final
        for p in range(sink, Sq):
            if p not in frozen:
                frozen[p] = (c.k_codes[0, 0, p].copy(), c.k_s[0, 0, p], c.k_z[0, 0, p])
        for p, (cc, ss, zz) in list(frozen.items())[-50:]:
            assert np.array_equal(c.k_codes[0, 0, p], cc) and c.k_s[0, 0, p] == ss


def test_capacity_overflow_leaves_sequence_untouched():
    c = ocache.Cache(2, 1, 128, 2, 1.0, 99.0, 4, 8, 4, capacity=20)
    T = np.eye(128, dtype=np.float16)[None]
    x = np.ones((2, 15, 1, 128), dtype=np.float16)
    c.append(x, x, T)
    c.S[1] = 3                                  # pretend sequence 1 is shorter
    y = np.ones((2, 10, 1, 128), dtype=np.float16)
    c.append(y, y, T)
    assert c.overflowed[0] and not c.overflowed[1]
    assert int(c.S[0]) == 15 and int(c.S[1]) == 13


# ---------------------------------------------------------------- attention
def _plain_attention(q, k, v, scale):
    w = softmax(scale * (k.astype(np.float64) @ q.astype(np.float64)))
    return w @ v.astype(np.float64)


def test_compensation_preserves_attention_exactly():
    """q' . k' = q . k: with no quantization and no fp16 rounding of k', compensated
    attention equals attention on the raw keys (to 1e-10, far inside 1e-5)."""
    rng = np.random.default_rng(3)
    d, S, Hkv, g = 128, 200, 2, 4
    c = ocache.Cache(1, Hkv, d, 2, 1.0, 99.0, 4, 1000, 16, capacity=S, chunk_max=S,
                     store_dtype=np.float64)
    k = rng.standard_normal((1, S, Hkv, d)).astype(np.float16)
    v = rng.standard_normal((1, S, Hkv, d)).astype(np.float16)
    a = rng.standard_normal((Hkv, d, d))
    T = (a + 4 * np.eye(d)).astype(np.float16)          # invertible, far from orthogonal
    c.append(k, v, T)
    assert int(c.S_quant[0]) == 0
    q = rng.standard_normal((1, Hkv * g, d)).astype(np.float16)
    scale = 1 / np.sqrt(d)
    out = attention.decode(c, q, T, scale)
    for j in range(Hkv * g):
        ref = _plain_attention(q[0, j], k[0, :, j // g], v[0, :, j // g], scale)
        np.testing.assert_allclose(out[0, j], ref, rtol=0, atol=1e-10)


def test_windows_only_is_textbook_softmax_and_single_token():
    rng = np.random.default_rng(4)
    d = 128
    c = ocache.Cache(1, 1, d, 2, 1.0, 99.0, 4, 64, 16, capacity=100, chunk_max=1)
    T = np.eye(d, dtype=np.float16)[None]
    k = rng.standard_normal((1, 1, 1, d)).astype(np.float16)
    v = rng.standard_normal((1, 1, 1, d)).astype(np.float16)
    c.append(k, v, T)
    q = rng.standard_normal((1, 4, d)).astype(np.float16)
    out = attention.decode(c, q, T, 0.1)
    for j in range(4):
        np.testing.assert_array_equal(out[0, j], v[0, 0, 0].astype(np.float64))
    ks = rng.standard_normal((1, 40, 1, d)).astype(np.float16)
    vs = rng.standard_normal((1, 40, 1, d)).astype(np.float16)
    for t in range(40):
        c.append(ks[:, t:t + 1], vs[:, t:t + 1], T)
    assert int(c.S_quant[0]) == 0
    out = attention.decode(c, q, T, 0.1)
    K = np.concatenate([k[0, :, 0], ks[0, :, 0]])
    V = np.concatenate([v[0, :, 0], vs[0, :, 0]])
    for j in range(4):
        np.testing.assert_allclose(out[0, j], _plain_attention(q[0, j], K, V, 0.1), rtol=0, atol=1e-12)


def test_empty_sequence_gives_zeros():
    c = ocache.Cache(1, 1, 128, 2, 1.0, 99.0, 4, 64, 16, capacity=10)
    out = attention.decode(c, np.ones((1, 2, 128), np.float16), np.eye(128, dtype=np.float16)[None], 0.1)
    assert not out.any()


def test_bruteforce_tiny_quantized_cache():
    """Tiny shape (512 tokens, 1 KV head, GQA 4, sink 4 + keep 32): the oracle's decode
    equals a brute-force recomputation that unpacks packed bytes, un-transforms the keys
    with a linear solve (instead of compensating the query) and uses scipy's softmax."""
    rng = np.random.default_rng(0)
    d, S, g = 128, 512, 4
    c = ocache.Cache(1, 1, d, 2, 1.0, 99.0, 4, 32, 16, capacity=S, chunk_max=1)
    k = rng.standard_normal((1, S, 1, d))
    k[..., [3, 50, 77, 101]] *= 20
    k = k.astype(np.float16)
    v = rng.standard_normal((1, S, 1, d)).astype(np.float16)
    qr, r = np.linalg.qr(rng.standard_normal((d, d)))
    T = ((qr * np.sign(np.diag(r))) * rng.uniform(0.5, 2, d))[None].astype(np.float16)
    for t0 in range(0, S, 16):
        c.append(k[:, t0:t0 + 16], v[:, t0:t0 + 16], T)
    Sq = int(c.S_quant[0])
    assert Sq > 400
    q = rng.standard_normal((1, g, d)).astype(np.float16)
    out = attention.decode(c, q, T, 1 / np.sqrt(d))
    # brute force
    kp16 = c.k_store[0, 0, :S].astype(np.float64)
    v16 = c.v_store[0, 0, :S].astype(np.float64)
    khat, vhat = kp16.copy(), v16.copy()
    for p in range(4, Sq):
        for arr, codes, s, z in ((khat, c.k_codes, c.k_s, c.k_z), (vhat, c.v_codes, c.v_s, c.v_z)):
            cc = quantizer.unpack(quantizer.pack(codes[0, 0, p], 2), 2).astype(np.float64)
            arr[p] = float(z[0, 0, p]) + float(s[0, 0, p]) * cc
    k_orig = np.linalg.solve(T[0].astype(np.float64), khat.T).T
    for j in range(g):
        w = softmax((k_orig @ q[0, j].astype(np.float64)) / np.sqrt(d))
        np.testing.assert_allclose(out[0, j], w @ vhat, rtol=0, atol=1e-9)
    # sanity: the fp16 k' really is T k rounded once
    kd = T[0].astype(np.float64) @ k[0, :, 0].astype(np.float64).T
    np.testing.assert_array_equal(kp16[S - 1], kd[:, S - 1].astype(np.float16).astype(np.float64))
