"""Query compensation and exact-softmax decode attention (oracle).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Source: "WUSH-KV: KV Cache Quantization with Data-Adaptive Transforms",
§4.1 (grouped-query attention re-evaluated at every new length S over the
cached K_h, V_h; its Eq. 2 was lost, so the standard scaled-dot-product form
softmax(q . k / sqrt(d)) is taken), §1 and §4.2 (the key transform's
query-side compensation is applied after normalisation and RoPE; with
k' = T_K k the compensated query is q' = T_K^{-T} q, so q' . k' = q . k),
§4.5 (the value transform is folded into the weights, so the output stays in
the value-transform basis) and §4.4 (attention reads the fp16 sink and recent
windows and the dequantized middle region; a new chunk is first appended in
full precision and is used to compute its own attention output, before the
flush quantizes it).

Query head j reads KV head floor(j / g), g = H_q / H_kv.  All arithmetic is
float64; the inverse of T_K is LAPACK's (numpy.linalg.inv).
"""
from __future__ import annotations

import numpy as np


def compensation(T_K: np.ndarray) -> np.ndarray:
    """T_K^{-T} in float64 from the stored (fp16) T_K: [..., d, d]."""
    return np.swapaxes(np.linalg.inv(T_K.astype(np.float64)), -1, -2)


def softmax_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float):
    """Exact softmax attention of one query: q [d], K [S, d], V [S, d] -> (o [d], m, l).

    m = max logit, l = sum exp(logit - m).
    """
    x = scale * (K @ q)
    m = x.max()
    w = np.exp(x - m)
    l = w.sum()
    return (w @ V) / l, m, l


def decode(cache, q: np.ndarray, T_K: np.ndarray, softmax_scale: float) -> np.ndarray:
    """Decode attention of one query per sequence: q fp16 [B, H_q, d] -> float64 [B, H_q, d].

    A sequence with S == 0 yields zeros (nothing to attend to).
    """
    B, Hq, d = q.shape
    g = Hq // cache.H
    Tinv_T = compensation(T_K)
    out = np.zeros((B, Hq, d), dtype=np.float64)
    for b in range(B):
        if int(cache.S[b]) == 0:
            continue
        for h in range(cache.H):
            K = cache.keys_hat(b, h)
            V = cache.values_hat(b, h)
            for j in range(h * g, (h + 1) * g):
                qc = Tinv_T[h] @ q[b, j].astype(np.float64)
                out[b, j], _, _ = softmax_attention(qc, K, V, softmax_scale)
    return out


def chunk_decode(cache, q: np.ndarray, T_K: np.ndarray, softmax_scale: float) -> np.ndarray:
    """Attention of a just-appended chunk's own queries (§4.4): q fp16 [B, n, H_q, d] holds
    the queries of the n newest positions S - n .. S - 1 of every sequence; query t of the
    chunk sits at position S - n + t and, as in any causal decoder, attends to the cached
    positions 0 .. S - n + t only.  Returns float64 [B, n, H_q, d].

    The cache must hold the chunk already (it was appended before its attention runs).
    """
    B, n, Hq, d = q.shape
    g = Hq // cache.H
    Tinv_T = compensation(T_K)
    out = np.zeros((B, n, Hq, d), dtype=np.float64)
    for b in range(B):
        S = int(cache.S[b])
        for h in range(cache.H):
            K = cache.keys_hat(b, h)
            V = cache.values_hat(b, h)
            for t in range(n):
                last = S - n + t  # the query's own position: the newest one it may see
                for j in range(h * g, (h + 1) * g):
                    qc = Tinv_T[h] @ q[b, t, j].astype(np.float64)
                    out[b, t, j], _, _ = softmax_attention(qc, K[:last + 1], V[:last + 1], softmax_scale)
    return out
