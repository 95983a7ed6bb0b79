"""Per-head RMSNorm and rotary position embedding of queries and keys (oracle).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Source: "WUSH-KV: KV Cache Quantization with Data-Adaptive Transforms", §4.1 (keys are
cached after head-wise normalisation and RoPE) and §4.2 (the key transform and the
query compensation act on the post-RoPE vectors): the path's inputs are q and k after
the per-head RMSNorm (where the model has one, as Qwen3 does) and RoPE.  The pages do
not restate either operation; the textbook definitions are taken:

* RMSNorm over the head dimension: y = x / sqrt(mean(x^2) + eps) * gain;
* RoPE with rotate-half pairing: dimension i < d/2 is paired with i + d/2 and the pair
  is rotated by the angle pos * theta^(-2i/d);
* the result is rounded once to fp16 (the format of the path's inputs); everything
  before that rounding is exact float64 here.
"""
from __future__ import annotations

import numpy as np


def rmsnorm(x: np.ndarray, gain=None, eps: float = 1e-6) -> np.ndarray:
    """x [..., d] float64 -> x / sqrt(mean(x^2) + eps) * gain (gain [d] or None = 1)."""
    x = np.asarray(x, dtype=np.float64)
    y = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    if gain is not None:
        y = y * np.asarray(gain, dtype=np.float64)
    return y


def rope_angles(pos, d: int, theta: float) -> np.ndarray:
    """Rotation angles [..., d/2] of positions `pos` (array): pos * theta^(-2i/d)."""
    i = np.arange(d // 2, dtype=np.float64)
    inv_freq = float(theta) ** (-2.0 * i / d)
    return np.asarray(pos, dtype=np.float64)[..., None] * inv_freq


def rope(x: np.ndarray, pos, theta: float) -> np.ndarray:
    """Rotate-half RoPE of x [..., d] at positions pos (broadcast over x's leading dims)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    h = d // 2
    ang = rope_angles(pos, d, theta)
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :h], x[..., h:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def prepare(x_fp16: np.ndarray, pos, theta: float, gain=None, eps: float = 1e-6,
            norm: bool = False) -> np.ndarray:
    """The path's input from a raw projection output: RMSNorm (if norm), RoPE at pos,
    rounded once to fp16.  x_fp16 [..., d]; pos broadcast against x's leading dims."""
    x = np.asarray(x_fp16, dtype=np.float64)
    if norm:
        x = rmsnorm(x, gain, eps)
    return rope(x, pos, theta).astype(np.float16)
