"""KV cache with full-precision sink and recent windows (oracle).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Source: "WUSH-KV: KV Cache Quantization with Data-Adaptive Transforms",
§4.1 (each new token appends one column to K_h and V_h; keys are cached after
head-wise normalisation and RoPE), §4.2 and §1 (the key transform acts on the
post-RoPE key: k' = T_K k), §4.5 (the value transform is folded into the
weights, so values arrive already transformed and are stored as given), and
§4.4 "Full-Precision Cache Window" (Algorithm 2, whose body the pages lost;
restated here from the prose):

* the first S_sink positions stay in full precision for good;
* of the remaining positions the newest S_keep form a rolling full-precision
  window;
* a new chunk is first appended in full precision and serves its own attention;
  then the largest multiple of S_flush among the entries outside both windows,
  under the current length S, is quantized;
* S_quant is the inclusive right boundary (1-based) of the quantized middle
  region, 0 for an empty cache.  With 0-based positions the quantized region is
  [S_sink, S_quant) once S_quant > 0.

Flush under a length S (one step of Algorithm 2):
    lo0 = max(S_quant, S_sink); e = S - S_keep - lo0
    if e >= S_flush: quantize [lo0, lo0 + floor(e / S_flush) * S_flush); advance S_quant.

Call order (the reading the library shares): ``append(n)`` with n <= chunk_max
first runs the flush that closes the previous chunk (its attention has been
computed by then), then stores the new chunk in full precision; so a decode
query issued after ``append`` sees the chunk unquantized, as the pages order it.
A chunk larger than chunk_max is stored and flushed at once (its own attention
is not part of this path).
"""
from __future__ import annotations

import numpy as np

from . import quantizer


class Cache:
    """One attention module's cache: B sequences x H_kv KV heads x capacity positions.

    Holds every position's full-precision k' and v (fp16, or float64 with
    ``store_dtype=np.float64`` for the exact-compensation pin), and codes plus
    (s, z) for quantized positions.
    """

    def __init__(self, batch, n_kv_heads, head_dim, bits, p_lo, p_hi,
                 s_sink, s_keep, s_flush, capacity, chunk_max=1,
                 store_dtype=np.float16, quantize_fn=None):
        self.B, self.H, self.d = batch, n_kv_heads, head_dim
        self.bits, self.p_lo, self.p_hi = bits, p_lo, p_hi
        self.S_sink, self.S_keep, self.S_flush = s_sink, s_keep, s_flush
        self.capacity, self.chunk_max = capacity, chunk_max
        self.store_dtype = store_dtype
        # the per-token quantizer: x fp16 [..., d] -> (codes, s, z); the percentile-clipped
        # affine one unless another is given (e.g. quest.quantize)
        self.quantize_fn = quantize_fn or (lambda x: quantizer.quantize(x, self.bits, self.p_lo, self.p_hi))
        self.S = np.zeros(batch, dtype=np.int64)
        self.S_quant = np.zeros(batch, dtype=np.int64)
        shape = (batch, n_kv_heads, capacity, head_dim)
        self.k_store = np.zeros(shape, dtype=store_dtype)
        self.v_store = np.zeros(shape, dtype=store_dtype)
        self.k_codes = np.zeros(shape, dtype=np.uint8)
        self.v_codes = np.zeros(shape, dtype=np.uint8)
        self.k_s = np.zeros(shape[:3], dtype=np.float16)
        self.k_z = np.zeros(shape[:3], dtype=np.float16)
        self.v_s = np.zeros(shape[:3], dtype=np.float16)
        self.v_z = np.zeros(shape[:3], dtype=np.float16)
        self.overflowed = np.zeros(batch, dtype=bool)

    # -- Algorithm 2 ---------------------------------------------------------
    def flush(self, b: int, S: int) -> None:
        """Quantize the largest multiple of S_flush outside both windows under length S."""
        lo0 = max(int(self.S_quant[b]), self.S_sink)
        e = S - self.S_keep - lo0
        if e < self.S_flush:
            return
        n = (e // self.S_flush) * self.S_flush
        sl = slice(lo0, lo0 + n)
        for store, codes, s_arr, z_arr in ((self.k_store, self.k_codes, self.k_s, self.k_z),
                                           (self.v_store, self.v_codes, self.v_s, self.v_z)):
            x = store[b, :, sl].astype(np.float16)
            c, s, z = self.quantize_fn(x)
            codes[b, :, sl] = c
            s_arr[b, :, sl] = s
            z_arr[b, :, sl] = z
        self.S_quant[b] = lo0 + n

    def transform_keys(self, k_new: np.ndarray, T_K: np.ndarray) -> np.ndarray:
        """k' = T_K k per token and KV head, in float64: k_new [n, H, d] -> [n, H, d]."""
        T = T_K.astype(np.float64)
        k = k_new.astype(np.float64)
        return np.einsum("hri,nhi->nhr", T, k)

    def append(self, k_new: np.ndarray, v_new: np.ndarray, T_K: np.ndarray) -> None:
        """Append a chunk to every sequence: k_new, v_new fp16 [B, n, H_kv, d]; T_K fp16 [H_kv, d, d].

        A sequence whose length would exceed the capacity is left untouched and
        flagged in ``overflowed``.
        """
        n = k_new.shape[1]
        for b in range(self.B):
            S = int(self.S[b])
            if S + n > self.capacity:
                self.overflowed[b] = True
                continue
            if n <= self.chunk_max:
                self.flush(b, S)
            kp = self.transform_keys(k_new[b], T_K).astype(self.store_dtype)
            self.k_store[b, :, S:S + n] = np.transpose(kp, (1, 0, 2))
            self.v_store[b, :, S:S + n] = np.transpose(v_new[b].astype(self.store_dtype), (1, 0, 2))
            self.S[b] = S + n
            if n > self.chunk_max:
                self.flush(b, S + n)

    # -- views -----------------------------------------------------------------
    def is_quantized(self, b: int) -> np.ndarray:
        """Boolean [S] mask of quantized positions of sequence b."""
        S = int(self.S[b])
        p = np.arange(S)
        return (p >= self.S_sink) & (p < int(self.S_quant[b]))

    def keys_hat(self, b: int, h: int) -> np.ndarray:
        """Keys as attention reads them, float64 [S, d]: stored k' in the windows, z + s c elsewhere."""
        return self._view(b, h, self.k_store, self.k_codes, self.k_s, self.k_z)

    def values_hat(self, b: int, h: int) -> np.ndarray:
        """Values as attention reads them, float64 [S, d]."""
        return self._view(b, h, self.v_store, self.v_codes, self.v_s, self.v_z)

    def _view(self, b, h, store, codes, s_arr, z_arr):
        S = int(self.S[b])
        out = store[b, h, :S].astype(np.float64)
        q = self.is_quantized(b)
        if q.any():
            out[q] = quantizer.dequantize(codes[b, h, :S][q], s_arr[b, h, :S][q], z_arr[b, h, :S][q])
        return out
