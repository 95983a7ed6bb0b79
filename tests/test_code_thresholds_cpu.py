"""The 2-bit quantizer in the kernels takes each code as #{k : x >= X_k}, with per-row fp16
thresholds X_k instead of a division per value (quantize.cuh, code_threshold).  This test
re-derives, on the CPU, the two facts that make that exact against the reading's code
c = clamp(rint_even(fl32(fl32(x - z) / s)), 0, 2^b - 1) (the percentile-clipped affine
quantizer of "WUSH-KV: KV Cache Quantization with Data-Adaptive Transforms", §5.3):

* in t = fl32(x - z): c >= k iff t >= T_k, T_k = (k - 1/2) s for even k and the next fp32
  value above it for odd k -- for every positive finite fp16 scale s and k <= 15;
* in x: the smallest fp16 x with fl32(x - z) >= T_k is the fp16 value nearest z + mid
  (mid = the midpoint below T_k, exact in double), moved by at most one fp16 step -- for
  every finite fp16 z against a sample of scales.
"""
import numpy as np

F32, F16 = np.float32, np.float16


def _code_ge(t, s, k):
    return np.rint((t / s).astype(F32)) >= k  # numpy division is correctly rounded; rint ties to even


def _threshold_t(s, k):
    e = (F32(k - 0.5) * s).astype(F32)
    return e if k % 2 == 0 else np.nextafter(e, F32(np.inf)).astype(F32)


def test_t_thresholds_closed_form_all_scales():
    s = np.arange(1, 0x7C00, dtype=np.uint16).view(F16).astype(F32)
    for k in range(1, 16):
        e = (F32(k - 0.5) * s).astype(F32)
        assert np.all(e.astype(np.float64) == (k - 0.5) * s.astype(np.float64))  # the product is exact
        T = _threshold_t(s, k)
        below = np.nextafter(T, F32(-np.inf)).astype(F32)
        assert np.all(_code_ge(T, s, k)) and not np.any(_code_ge(below, s, k)), k


def _order_key(b):
    b = b.astype(np.int64)
    return np.where(b >= 0x8000, 0xFFFF - b, b + 0x8000)


def _step(b, d):
    k = np.clip(_order_key(b) + d, 0, 0xFFFF)
    return np.where(k >= 0x8000, k - 0x8000, 0xFFFF - k).astype(np.uint16)


def test_x_thresholds_one_step_from_the_nearest():
    zb = np.arange(0, 0x10000, dtype=np.uint16)
    zb = zb[np.isfinite(zb.view(F16))]
    z64 = zb.view(F16).astype(np.float64)
    z32 = zb.view(F16).astype(F32)
    rng = np.random.default_rng(7)
    scales = np.concatenate([rng.integers(1, 0x7C00, 40), [1, 0x3FF, 0x400, 0x3C00, 0x7BFF]]).astype(np.uint16)
    for s in scales.view(F16).astype(F32):
        for k in (1, 2, 3, 8, 15):
            T = _threshold_t(np.array([s], F32), k)[0]
            mid = 0.5 * (np.float64(T) + np.float64(np.nextafter(T, F32(-np.inf))))
            incl = (np.array(T).view(np.uint32) & 1) == 0

            def reach_exact(xb):
                y = xb.view(F16).astype(np.float64) - z64
                return (y >= mid) if incl else (y > mid)

            def reach_fp32(xb):
                with np.errstate(invalid="ignore", over="ignore"):
                    return (xb.view(F16).astype(F32) - z32).astype(F32) >= T

            with np.errstate(over="ignore"):
                v = (z64 + mid).astype(F16).view(np.uint16)
            r = reach_exact(v)
            p = _step(v, -1)
            X = np.where(r & reach_exact(p), p, v)
            X = np.where(~r, _step(v, 1), X)
            is_inf = X.view(F16).astype(F32) == np.inf
            assert np.all(reach_fp32(X) | is_inf), (s, k)
            assert not np.any(reach_fp32(_step(X, -1))), (s, k)
