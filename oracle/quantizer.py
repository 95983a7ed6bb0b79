"""Per-token percentile-clipped asymmetric affine quantizer (oracle).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Source: "WUSH-KV: KV Cache Quantization with Data-Adaptive Transforms",
§5.3 "Downstream Benchmarks" (the end-to-end quantizer combines percentile
clipping with asymmetric affine scaling and an adaptive zero point), §1
(per-token clipped quantizers), and the cnshai.top post section "WUSH-KV:
quantize in the right coordinate system" (OSCAR-style percentile-clipped affine
quantization).  The pages print no formula for it; the readings taken here:

* a group is one token's head vector (d = 128 values, "per-token");
* the clipping range is [lo, hi] with lo / hi the p_lo-th / p_hi-th percentile
  of the group, linear interpolation between order statistics at rank
  p/100 * (d - 1);
* asymmetric affine: zero point z = lo, step s = (hi - lo) / (2^b - 1), both
  stored as fp16; the codes are computed from the stored (rounded) s and z;
* code c = clamp(round_half_even((x - z) / s), 0, 2^b - 1); s == 0 gives c = 0;
* dequantized value x_hat = z + s * c;
* every fp32 step is one IEEE operation, rounded on its own (no fused
  multiply-add), so the decisions that turn floats into codes are fixed.

Packing (the layout of ``include/wushkv.h``): code j of a group sits in byte
floor(j * b / 8) at bit offset (j * b) mod 8.
"""
from __future__ import annotations

import numpy as np


def percentile_rank(p: float, d: int):
    """Rank split of the p-th percentile of d sorted values: (i, f).

    pos = p/100 * (d-1) in double; i = floor(pos); f = fp32(pos - i).
    """
    pos = (float(p) / 100.0) * float(d - 1)
    i = int(np.floor(pos))
    f = np.float32(pos - i)
    return i, f


def percentile_fp32(x_sorted: np.ndarray, i: int, f: np.float32) -> np.ndarray:
    """Linear interpolation between order statistics, in fp32.

    P = s[i] + f * (s[i+1] - s[i]), three separately rounded fp32 operations,
    with s[d] read as s[d-1] (the 100th percentile is the maximum, plus +0).
    Written this way the result never depends on how a sort orders -0 and +0.
    x_sorted: float32 [..., d] ascending.
    """
    d = x_sorted.shape[-1]
    a = x_sorted[..., i]
    b = x_sorted[..., min(i + 1, d - 1)]
    diff = np.subtract(b, a, dtype=np.float32)
    step = np.multiply(np.float32(f), diff, dtype=np.float32)
    return np.add(a, step, dtype=np.float32)


def clip_range(x_fp16: np.ndarray, p_lo: float, p_hi: float):
    """(lo, hi) fp32 clipping range of every group of x: fp16 [..., d]."""
    d = x_fp16.shape[-1]
    xs = np.sort(x_fp16.astype(np.float32), axis=-1)
    i_lo, f_lo = percentile_rank(p_lo, d)
    i_hi, f_hi = percentile_rank(p_hi, d)
    return percentile_fp32(xs, i_lo, f_lo), percentile_fp32(xs, i_hi, f_hi)


def affine_params(x_fp16: np.ndarray, bits: int, p_lo: float, p_hi: float):
    """Stored step and zero point (s, z), both fp16 [...], of every group."""
    lo, hi = clip_range(x_fp16, p_lo, p_hi)
    levels = np.float32(2 ** bits - 1)
    scale32 = np.divide(np.subtract(hi, lo, dtype=np.float32), levels, dtype=np.float32)
    return scale32.astype(np.float16), lo.astype(np.float16)


def quantize_codes(x_fp16: np.ndarray, s: np.ndarray, z: np.ndarray, bits: int) -> np.ndarray:
    """Codes uint8 [..., d] of x under the stored (s, z) of its group."""
    x32 = x_fp16.astype(np.float32)
    s32 = s.astype(np.float32)[..., None]
    z32 = z.astype(np.float32)[..., None]
    t = np.subtract(x32, z32, dtype=np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.divide(t, s32, dtype=np.float32)
    c = np.clip(np.rint(q), 0, 2 ** bits - 1)
    c = np.where(s32 == 0, 0, c)
    return c.astype(np.uint8)


def quantize(x_fp16: np.ndarray, bits: int, p_lo: float, p_hi: float):
    """Quantize every group of x: returns (codes uint8 [..., d], s fp16 [...], z fp16 [...])."""
    x_fp16 = np.asarray(x_fp16, dtype=np.float16)
    s, z = affine_params(x_fp16, bits, p_lo, p_hi)
    return quantize_codes(x_fp16, s, z, bits), s, z


def dequantize(codes: np.ndarray, s: np.ndarray, z: np.ndarray) -> np.ndarray:
    """x_hat = z + s * c in float64: [..., d]."""
    return z.astype(np.float64)[..., None] + s.astype(np.float64)[..., None] * codes.astype(np.float64)


def pack(codes: np.ndarray, bits: int) -> np.ndarray:
    """Bit-pack codes [..., d] into bytes [..., d*bits/8]; code j -> byte j*b//8, bit (j*b)%8."""
    d = codes.shape[-1]
    per = 8 // bits
    c = codes.astype(np.uint16).reshape(codes.shape[:-1] + (d // per, per))
    out = np.zeros(codes.shape[:-1] + (d // per,), dtype=np.uint16)
    for k in range(per):
        out |= c[..., k] << (k * bits)
    return out.astype(np.uint8)


def unpack(packed: np.ndarray, bits: int) -> np.ndarray:
    """Inverse of ``pack``: bytes [..., n] -> codes uint8 [..., n*8/bits]."""
    per = 8 // bits
    mask = (1 << bits) - 1
    p = packed.astype(np.uint16)
    parts = [(p >> (k * bits)) & mask for k in range(per)]
    return np.stack(parts, axis=-1).reshape(packed.shape[:-1] + (packed.shape[-1] * per,)).astype(np.uint8)
