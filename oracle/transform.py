"""Structured key transform: the normalised Walsh-Hadamard matrix (oracle).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Source: "WUSH-KV: KV Cache Quantization with Data-Adaptive Transforms", the Hadamard
baseline of its transform comparison and the future-work note on cheaper structured
transforms (§6).  The normalised Hadamard matrix H (Sylvester construction, scaled by
1/sqrt(d)) is orthonormal and symmetric, so used as T_K it is its own compensation:
T_K^{-T} = H.  The oracle's cache and attention take it as an ordinary float64 T_K.
"""
from __future__ import annotations

import numpy as np


def hadamard(d: int = 128) -> np.ndarray:
    """Normalised Sylvester Hadamard matrix, float64 [d, d]: H[r, i] = (-1)^popcount(r & i) / sqrt(d)."""
    assert d > 0 and d & (d - 1) == 0
    h = np.ones((1, 1))
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h / np.sqrt(d)
