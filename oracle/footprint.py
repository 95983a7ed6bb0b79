"""Cache-size arithmetic (oracle).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Source: cnshai.top post "kv-cache-quantization-fp8-training", section "The KV
cache is the wall": per token the cache holds K and V for every layer and KV
head; at fp16 each value costs 2 bytes; at b bits, b/8 bytes (codes only; the
per-token step and zero point are not counted in the pages' figure).  Also
"WUSH-KV: KV Cache Quantization with Data-Adaptive Transforms", §4.5 "Storage
and Computation Costs": 2 * n_layer * n_kv * d * S cached elements.
"""
from __future__ import annotations


def values_per_token(n_layer: int, n_kv: int, d: int) -> int:
    """K and V elements cached per token: 2 * n_layer * n_kv * d."""
    return 2 * n_layer * n_kv * d


def cached_elements(n_layer: int, n_kv: int, d: int, seq_len: int) -> int:
    """Elements cached for a sequence of length S."""
    return values_per_token(n_layer, n_kv, d) * seq_len


def bytes_fp16(n_layer: int, n_kv: int, d: int, seq_len: int = 1) -> int:
    """Bytes at fp16 (2 bytes per element)."""
    return 2 * cached_elements(n_layer, n_kv, d, seq_len)


def bytes_codes(n_layer: int, n_kv: int, d: int, seq_len: int, bits: int) -> int:
    """Bytes of the packed codes alone at b bits per element."""
    return cached_elements(n_layer, n_kv, d, seq_len) * bits // 8
