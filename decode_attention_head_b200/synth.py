"""Seeded synthetic inputs for the WUSH-KV append + decode-attention path.

This module only draws numbers.  It holds none of the method's arithmetic (no
key transform application, no quantizer, no attention): it produces the tensors
that arrive at the path's boundary, shaped like the workloads the WUSH-KV pages
describe ("WUSH-KV: KV Cache Quantization with Data-Adaptive Transforms",
§4.1 "KV Cache in Grouped-Query Attention" and §5; and the cnshai.top post
"kv-cache-quantization-fp8-training", section "The KV cache is the wall").

What arrives at the boundary (all fp16 unless stated):

* keys ``k``: post-normalisation, post-RoPE key head vectors.  Drawn N(0, 1),
  four seeded outlier channels per KV head scaled x20, then (Qwen3-shaped
  workloads only) a unit-gain per-head RMSNorm, then rotate-half RoPE at the
  token's position.  Keys are stored after head-wise normalisation and RoPE
  (§4.1), so those two steps shape the input and are not part of the path.
* values ``v``: already in the value-transform basis (the value transform is
  folded into the projection weights, §4.5), so they are taken as given:
  Student-t(5) for the model-shaped workloads, N(0,1) with outlier channels for
  the tiny one.
* queries ``q``: N(0,1) (+ RMSNorm for Qwen3) and RoPE at the decode position.
* the calibration artefacts of one KV head: ``T_K`` = Haar-random orthogonal
  matrix x diag(U[0.5, 2]) rounded to fp16 (the key transform is a full
  invertible d x d matrix, §2 and §4.2).  Its inverse-transpose is *not*
  computed here; the library and the oracle each derive their own.

Every unit (layer, sequence, KV head) has its own counter-derived seed, so any
unit can be regenerated alone, on any device, without drawing the others.  The
CPU and CUDA generators of torch produce different streams; tests that compare
against the oracle draw on the CPU.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

HEAD_DIM = 128

# stream tags mixed into the per-unit seed
_TAG_K, _TAG_V, _TAG_Q, _TAG_T, _TAG_OUT_K, _TAG_OUT_V = 1, 2, 3, 4, 5, 6


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and distribution of one synthetic workload."""

    name: str
    n_layers: int
    batch: int
    n_kv_heads: int
    n_q_heads: int
    context: int                 # cached positions when the decode query runs
    bits: int
    p_lo: float
    p_hi: float
    s_sink: int
    s_keep: int
    s_flush: int
    rope_theta: Optional[float]  # None: no RoPE
    qk_rmsnorm: bool
    v_dist: str                  # "normal_outliers" | "student_t5"
    seed: int
    prefill_chunk: int = 0       # >0: the last `prefill_chunk` tokens arrive as one append
    head_dim: int = HEAD_DIM

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads


WORKLOADS = {
    # tiny parity case: 512 cached tokens, one KV head, GQA 4
    "tiny": Workload("tiny", 1, 1, 1, 4, 512, 2, 1.0, 99.0, 4, 32, 16,
                     None, False, "normal_outliers", 0),
    # Llama-3-8B-shaped attention layer at 32K context, batch 8
    "llama3-8b-layer": Workload("llama3-8b-layer", 1, 8, 8, 32, 32768, 2, 1.0, 99.0,
                                4, 128, 16, 500000.0, False, "student_t5", 1),
    # Qwen3-8B-shaped layer at 128K context, batch 1 (long-context bandwidth case)
    "qwen3-8b-layer": Workload("qwen3-8b-layer", 1, 1, 8, 32, 131072, 2, 1.0, 99.0,
                               4, 128, 16, 1000000.0, True, "student_t5", 2),
    # 32 layers x 32 KV heads MHA at 8K context, batch 64, 4-bit with 0.5/99.5 clip
    "mha-32l": Workload("mha-32l", 32, 64, 32, 32, 8192, 4, 0.5, 99.5,
                        4, 64, 16, 10000.0, False, "student_t5", 3),
    # 16,384-token chunk appended onto a 114,688-token cache, then decode at 131,072
    "prefill-append-decode": Workload("prefill-append-decode", 1, 4, 8, 64, 131072, 2,
                                      1.0, 99.0, 4, 128, 16, 1000000.0, False,
                                      "student_t5", 4, prefill_chunk=16384),
}


def unit_seed(seed: int, tag: int, layer: int = 0, b: int = 0, h: int = 0) -> int:
    """Counter-derived 63-bit seed for one stream of one unit (SplitMix64 mixing)."""
    x = (seed * 0x9E3779B97F4A7C15 + tag * 0xBF58476D1CE4E5B9 + layer * 0x94D049BB133111EB
         + b * 0x2545F4914F6CDD1D + h * 0x9E6C63D0676A9A99) & 0xFFFFFFFFFFFFFFFF
    x ^= x >> 30
    x = (x * 0xBF58476D1CE4E5B9) & 0xFFFFFFFFFFFFFFFF
    x ^= x >> 27
    x = (x * 0x94D049BB133111EB) & 0xFFFFFFFFFFFFFFFF
    x ^= x >> 31
    return x & 0x7FFFFFFFFFFFFFFF


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _rmsnorm(x: torch.Tensor, eps: float = 1e-6) -> torch.Tensor:
    return x * torch.rsqrt(x.pow(2).mean(dim=-1, keepdim=True) + eps)


def _rope(x: torch.Tensor, pos: torch.Tensor, theta: float) -> torch.Tensor:
    """Rotate-half RoPE; x [..., n, d] float32, pos [n] positions."""
    d = x.shape[-1]
    half = d // 2
    inv = theta ** (-torch.arange(0, half, dtype=torch.float64, device=x.device) * 2.0 / d)
    ang = pos.to(torch.float64)[:, None] * inv[None, :]
    cos = torch.cos(ang).to(torch.float32)
    sin = torch.sin(ang).to(torch.float32)
    x1, x2 = x[..., :half], x[..., half:]
    return torch.cat([x1 * cos - x2 * sin, x2 * cos + x1 * sin], dim=-1)


def _outlier_channels(wl: Workload, tag: int, layer: int, h: int) -> torch.Tensor:
    g = _gen("cpu", unit_seed(wl.seed, tag + 100, layer, 0, h))
    return torch.randperm(wl.head_dim, generator=g)[:4]


def _student_t5(n, d, g, device) -> torch.Tensor:
    z = torch.randn(n, d, generator=g, device=device)
    chi = torch.randn(5, n, d, generator=g, device=device).pow(2).sum(0)
    return z / torch.sqrt(chi / 5.0)


def keys(wl: Workload, layer: int, b: int, h: int, start: int, n: int,
         device="cpu") -> torch.Tensor:
    """Keys of positions [start, start+n) of unit (layer, b, h): fp16 [n, d].

    The draw for a position depends only on (unit, position block of 4096), so a
    sub-range can be regenerated alone.
    """
    return _unit_stream(wl, _TAG_K, layer, b, h, start, n, device)


def values(wl: Workload, layer: int, b: int, h: int, start: int, n: int,
           device="cpu") -> torch.Tensor:
    """Values of positions [start, start+n) of unit (layer, b, h): fp16 [n, d]."""
    return _unit_stream(wl, _TAG_V, layer, b, h, start, n, device)


_BLOCK = 4096


def _unit_stream(wl, tag, layer, b, h, start, n, device) -> torch.Tensor:
    d = wl.head_dim
    out = torch.empty(n, d, dtype=torch.float16, device=device)
    if n == 0:
        return out
    first, last = start // _BLOCK, (start + n - 1) // _BLOCK
    ch = _outlier_channels(wl, tag, layer, h).to(device)
    for blk in range(first, last + 1):
        g = _gen(device, unit_seed(wl.seed, tag, layer, b, h * 1_000_003 + blk))
        if tag == _TAG_V and wl.v_dist == "student_t5":
            x = _student_t5(_BLOCK, d, g, device)
        else:
            x = torch.randn(_BLOCK, d, generator=g, device=device)
            x[:, ch] *= 20.0
        if tag == _TAG_K:
            if wl.qk_rmsnorm:
                x = _rmsnorm(x)
            if wl.rope_theta is not None:
                pos = torch.arange(blk * _BLOCK, (blk + 1) * _BLOCK, device=device)
                x = _rope(x, pos, wl.rope_theta)
        lo = max(start, blk * _BLOCK)
        hi = min(start + n, (blk + 1) * _BLOCK)
        out[lo - start:hi - start] = x[lo - blk * _BLOCK:hi - blk * _BLOCK].to(torch.float16)
    return out


def queries(wl: Workload, layer: int, b: int, position: int, device="cpu") -> torch.Tensor:
    """Decode queries of sequence b at `position`: fp16 [H_q, d]."""
    g = _gen(device, unit_seed(wl.seed, _TAG_Q, layer, b, position))
    x = torch.randn(wl.n_q_heads, wl.head_dim, generator=g, device=device)
    if wl.qk_rmsnorm:
        x = _rmsnorm(x)
    if wl.rope_theta is not None:
        pos = torch.full((wl.n_q_heads,), position, device=device)
        x = _rope(x.unsqueeze(0), pos, wl.rope_theta).squeeze(0)
    return x.to(torch.float16)


def key_transform(wl: Workload, layer: int, h: int, identity: bool = False) -> torch.Tensor:
    """Calibration key transform T_K of (layer, KV head h): fp16 [d, d], acts on columns.

    Haar-random orthogonal (QR of a Gaussian with the sign of diag(R) folded in)
    times diag(U[0.5, 2]).
    """
    d = wl.head_dim
    if identity:
        return torch.eye(d, dtype=torch.float16)
    g = _gen("cpu", unit_seed(wl.seed, _TAG_T, layer, 0, h))
    a = torch.randn(d, d, generator=g, dtype=torch.float64)
    qm, r = torch.linalg.qr(a)
    qm = qm * torch.sign(torch.diagonal(r))[None, :]
    u = 0.5 + 1.5 * torch.rand(d, generator=g, dtype=torch.float64)
    return (qm * u[None, :]).to(torch.float16)


def key_transforms(wl: Workload, layer: int = 0, identity: bool = False) -> torch.Tensor:
    """T_K of every KV head of a layer: fp16 [H_kv, d, d]."""
    return torch.stack([key_transform(wl, layer, h, identity) for h in range(wl.n_kv_heads)])


def batch_tokens(wl: Workload, layer: int, start: int, n: int, device="cpu",
                 which: str = "k") -> torch.Tensor:
    """Keys or values of positions [start, start+n) for every (b, h): fp16 [B, n, H_kv, d]."""
    fn = keys if which == "k" else values
    out = torch.empty(wl.batch, n, wl.n_kv_heads, wl.head_dim, dtype=torch.float16, device=device)
    for b in range(wl.batch):
        for h in range(wl.n_kv_heads):
            out[b, :, h] = fn(wl, layer, b, h, start, n, device)
    return out


def batch_queries(wl: Workload, layer: int, position: int, device="cpu") -> torch.Tensor:
    """Decode queries of every sequence at `position`: fp16 [B, H_q, d]."""
    return torch.stack([queries(wl, layer, b, position, device) for b in range(wl.batch)])


def scaled(wl: Workload, **changes) -> Workload:
    """A copy of `wl` with some fields replaced (smaller parity cases of one shape)."""
    return dataclasses.replace(wl, **changes)


def default_softmax_scale(d: int = HEAD_DIM) -> float:
    return 1.0 / math.sqrt(d)


def bulk_tokens(wl: Workload, layer: int, start: int, n: int, device="cpu", which: str = "k",
                gen_seed: Optional[int] = None) -> torch.Tensor:
    """Keys or values of positions [start, start+n) for all (b, h) in one draw: fp16 [B, n, H_kv, d].

    Same recipe as `keys` / `values` (outlier channels per KV head, RMSNorm, RoPE at the
    positions, Student-t(5) values), but one generator per call, so it is fast on a GPU
    and not element-identical to the per-unit streams.
    """
    tag = _TAG_K if which == "k" else _TAG_V
    seed = unit_seed(wl.seed, tag + 50, layer, start, n) if gen_seed is None else gen_seed
    g = _gen(device, seed)
    B, H, d = wl.batch, wl.n_kv_heads, wl.head_dim
    if tag == _TAG_V and wl.v_dist == "student_t5":
        z = torch.randn(B, n, H, d, generator=g, device=device)
        chi = torch.zeros_like(z)
        for _ in range(5):
            chi.add_(torch.randn(B, n, H, d, generator=g, device=device).pow_(2))
        x = z.div_(chi.div_(5.0).sqrt_())
    else:
        x = torch.randn(B, n, H, d, generator=g, device=device)
        for h in range(H):
            ch = _outlier_channels(wl, tag, layer, h).to(device)
            x[:, :, h, ch] *= 20.0
    if tag == _TAG_K:
        if wl.qk_rmsnorm:
            x = _rmsnorm(x)
        if wl.rope_theta is not None:
            pos = torch.arange(start, start + n, device=device)
            x = _rope(x.transpose(1, 2), pos, wl.rope_theta).transpose(1, 2)
    return x.to(torch.float16).contiguous()


def bulk_queries(wl: Workload, layer: int, position: int, device="cpu", gen_seed: Optional[int] = None):
    """Decode queries of every sequence at `position` in one draw: fp16 [B, H_q, d]."""
    seed = unit_seed(wl.seed, _TAG_Q + 50, layer, position) if gen_seed is None else gen_seed
    g = _gen(device, seed)
    x = torch.randn(wl.batch, wl.n_q_heads, wl.head_dim, generator=g, device=device)
    if wl.qk_rmsnorm:
        x = _rmsnorm(x)
    if wl.rope_theta is not None:
        pos = torch.full((wl.n_q_heads,), position, device=device)
        x = _rope(x, pos, wl.rope_theta)
    return x.to(torch.float16)
