"""RMS-scaled symmetric integer quantizer, the QuEST-style alternative (oracle).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Source: "WUSH-KV: KV Cache Quantization with Data-Adaptive Transforms", §4.3 (the
analysis uses QuEST INT with rounding inside the clipping range) and Appendix B.3 (the
scalar grid: the 2^b equally spaced levels from -alpha to alpha, spacing
Delta = 2 alpha / (2^b - 1), with alpha_b the clipping endpoint that is optimal for a
standard Gaussian; QuEST itself scales that grid by each group's RMS).  The pages lost the
quantizer's own equation (Eq. 5), so this is a reading:

* group = one token's head vector (d = 128), sigma = RMS of the group;
* the grid is -alpha*sigma + k * 2*alpha*sigma / (2^b - 1), k = 0 .. 2^b - 1, i.e. the
  affine quantizer of ``quantizer.py`` with z = fp16(-alpha*sigma) and
  s = fp16(2*alpha/(2^b-1) * sigma), codes from the stored s and z as there;
* alpha_b minimises the mean squared error of that grid on N(0,1), found numerically;
* sigma^2 is summed in fp32 in a fixed order (four groups of 32 consecutive elements,
  each summed left to right, then (g0 + g1) + (g2 + g3)), divided by 128, and its fp32
  square root taken, every operation rounded on its own, so the decisions are fixed;
* the constants 2*alpha/(2^b-1) and alpha are rounded to fp32 once.
"""
from __future__ import annotations

import numpy as np
from scipy import integrate, optimize, stats

from . import quantizer


def grid_mse(alpha: float, bits: int) -> float:
    """E[(zeta - Q_alpha(zeta))^2] for zeta ~ N(0,1), Q_alpha the nearest of the 2^b levels
    equally spaced on [-alpha, alpha] (values beyond the ends clip to them)."""
    n = 2 ** bits
    levels = np.linspace(-alpha, alpha, n)
    edges = np.concatenate([[-np.inf], (levels[:-1] + levels[1:]) / 2, [np.inf]])
    total = 0.0
    for k in range(n):
        f = lambda z, c=levels[k]: (z - c) ** 2 * stats.norm.pdf(z)
        val, _ = integrate.quad(f, edges[k], edges[k + 1], epsabs=1e-13, epsrel=1e-12)
        total += val
    return total


def gaussian_optimal_alpha(bits: int) -> float:
    """The MSE-optimal clipping endpoint alpha_b of the b-bit symmetric grid on N(0,1)."""
    res = optimize.minimize_scalar(lambda a: grid_mse(a, bits), bounds=(0.5, 6.0), method="bounded",
                                   options={"xatol": 1e-10})
    return float(res.x)


def rms_fp32(x_fp16: np.ndarray) -> np.ndarray:
    """sigma of every group of x (fp16 [..., 128]) in the fixed fp32 order described above."""
    x = np.asarray(x_fp16, dtype=np.float32)
    sq = np.multiply(x, x, dtype=np.float32)
    g = []
    for j in range(4):
        acc = np.zeros(x.shape[:-1], dtype=np.float32)
        for i in range(32 * j, 32 * j + 32):
            acc = np.add(acc, sq[..., i], dtype=np.float32)
        g.append(acc)
    ss = np.add(np.add(g[0], g[1], dtype=np.float32), np.add(g[2], g[3], dtype=np.float32), dtype=np.float32)
    mean = np.divide(ss, np.float32(128.0), dtype=np.float32)
    return np.sqrt(mean, dtype=np.float32)


def params(x_fp16: np.ndarray, bits: int, alpha: float):
    """(s, z) fp16 [...] of every group of x."""
    sigma = rms_fp32(x_fp16)
    kb = np.float32(2.0 * alpha / (2 ** bits - 1))
    a32 = np.float32(alpha)
    s = np.multiply(kb, sigma, dtype=np.float32).astype(np.float16)
    z = np.multiply(-a32, sigma, dtype=np.float32).astype(np.float16)
    return s, z


def quantize(x_fp16: np.ndarray, bits: int, alpha: float):
    """(codes uint8 [..., 128], s fp16 [...], z fp16 [...]) of every group of x."""
    s, z = params(x_fp16, bits, alpha)
    return quantizer.quantize_codes(x_fp16, s, z, bits), s, z
