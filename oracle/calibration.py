"""Calibration statistics of the cached vectors: per-KV-head Gram matrices (oracle).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Source: "WUSH-KV: KV Cache Quantization with Data-Adaptive Transforms".
  - §3: the WUSH transform is built from M, the Gram matrix of the tensor being quantized.
  - Appendix B.1: M = X X^T, where each column of X is one quantization group.  For this
    cache's per-token quantizer a group is one token's 128-vector of one KV head, so
    M_h = sum_t x_{t,h} x_{t,h}^T.
  - §5.2, Setup: an unquantized forward pass accumulates, per KV head, the key Gram
    matrices (after RMS normalisation and RoPE) and the value Gram matrices.

The Gram matrix here is the plain sum over the tokens seen, not a mean.  The pages note
(§3) that the WUSH construction is invariant to a positive rescaling of M, so the
normalisation is immaterial.  Accumulating batch after batch, as a calibration pass
does, is repeated addition of this sum.
"""
from __future__ import annotations

import numpy as np


def gram(x) -> np.ndarray:
    """Per-head Gram matrices of a batch of cached vectors.

    x: [n_tokens, n_heads, d], any real dtype; fp16 inputs are widened exactly.
    Returns float64 [n_heads, d, d]: M_h = X_h X_h^T, with X_h = x[:, h, :]^T of shape
    d x n_tokens (tokens as columns, the pages' convention).
    """
    xd = np.asarray(x, dtype=np.float64)
    assert xd.ndim == 3, "x must be [n_tokens, n_heads, d]"
    n_tokens, n_heads, d = xd.shape
    out = np.zeros((n_heads, d, d))
    for h in range(n_heads):
        X = xd[:, h, :].T  # d x n_tokens
        out[h] = X @ X.T
    return out
