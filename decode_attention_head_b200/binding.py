"""ctypes binding of libwushkv (include/wushkv.h): argument marshalling only.

Every step of the append and decode-attention path runs in the library's CUDA
kernels; PyTorch only provides device memory and streams.  If the library is
missing the import of this module fails: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libwushkv.so")

OK, EINVAL, EUNSUPPORTED, ECUDA, ESINGULAR, ESCRATCH = 0, -1, -2, -3, -4, -5
STATIC_SCRATCH_BYTES = 8 << 20  # WUSHKV_STATIC_SCRATCH_BYTES
STATUS_OVERFLOW, STATUS_EMPTY, STATUS_TIMEOUT, STATUS_BADSTATE, STATUS_CHUNK_QUANTIZED = 1, 2, 4, 8, 16
_ERR = {EINVAL: "invalid argument", EUNSUPPORTED: "unsupported configuration", ECUDA: "CUDA launch failed",
        ESINGULAR: "singular key transform", ESCRATCH: "needs more than the static scratch array holds"}
SYMBOLS = ("wushkv_pack_layout", "wushkv_compensation", "wushkv_hadamard", "wushkv_append", "wushkv_decode_attn",
           "wushkv_chunk_attn", "wushkv_step", "wushkv_step_prep", "wushkv_decode_attn_static",
           "wushkv_gram_accumulate", "wushkv_decode_attn_test_timeout")


class Prep(ctypes.Structure):
    _fields_ = [("rope_theta", ctypes.c_float), ("q_norm_gain", ctypes.c_void_p), ("k_norm_gain", ctypes.c_void_p),
                ("norm_eps", ctypes.c_float)]


class Config(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("bits", ctypes.c_int32), ("capacity", ctypes.c_int32),
                ("s_sink", ctypes.c_int32), ("s_keep", ctypes.c_int32), ("s_flush", ctypes.c_int32),
                ("chunk_max", ctypes.c_int32), ("p_lo", ctypes.c_float), ("p_hi", ctypes.c_float),
                ("transform", ctypes.c_int32), ("quantizer", ctypes.c_int32), ("clip_alpha", ctypes.c_float)]


TRANSFORM_DENSE, TRANSFORM_HADAMARD = 0, 1
QUANT_PERCENTILE, QUANT_RMS = 0, 1
CODE_ORDER_CANONICAL, CODE_ORDER_VGROUP16 = 0, 1


class Layout(ctypes.Structure):
    _fields_ = [("codes_bytes", ctypes.c_size_t), ("params_bytes", ctypes.c_size_t),
                ("sink_bytes", ctypes.c_size_t), ("ring_bytes", ctypes.c_size_t),
                ("state_bytes", ctypes.c_size_t), ("workspace_bytes", ctypes.c_size_t),
                ("cap_alloc", ctypes.c_int32), ("ring_slots", ctypes.c_int32), ("code_bytes", ctypes.c_int32),
                ("n_splits", ctypes.c_int32), ("split_tokens", ctypes.c_int32), ("code_order", ctypes.c_int32),
                ("chunk_workspace_bytes", ctypes.c_size_t), ("decode_cluster", ctypes.c_int32),
                ("decode_interleave", ctypes.c_int32)]


class CacheBufs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("k_codes", "v_codes", "k_params", "v_params", "k_sink", "v_sink",
                                               "k_ring", "v_ring", "state")]


class WushKVError(RuntimeError):
    pass


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libwushkv.so not built ({LIB_PATH}); run decode_attention_head_b200.build.build()")
    lib = ctypes.CDLL(LIB_PATH)
    lib.wushkv_pack_layout.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(Layout)]
    lib.wushkv_compensation.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p]
    lib.wushkv_hadamard.argtypes = [ctypes.c_int32, ctypes.c_void_p]
    lib.wushkv_append.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(CacheBufs), ctypes.c_void_p,
                                  ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]
    lib.wushkv_decode_attn.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(CacheBufs), ctypes.c_void_p,
                                       ctypes.c_void_p, ctypes.c_float, ctypes.c_int32, ctypes.c_void_p,
                                       ctypes.c_void_p, ctypes.c_void_p]
    lib.wushkv_step.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(CacheBufs), ctypes.c_void_p, ctypes.c_void_p,
                                ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float,
                                ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    lib.wushkv_step_prep.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(CacheBufs), ctypes.c_void_p,
                                     ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.c_void_p, ctypes.c_float, ctypes.c_int32, ctypes.c_void_p,
                                     ctypes.c_void_p, ctypes.POINTER(Prep), ctypes.c_void_p]
    lib.wushkv_chunk_attn.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(CacheBufs), ctypes.c_void_p,
                                      ctypes.c_int32, ctypes.c_void_p, ctypes.c_float, ctypes.c_int32, ctypes.c_void_p,
                                      ctypes.c_void_p, ctypes.c_void_p]
    lib.wushkv_decode_attn_static.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(CacheBufs), ctypes.c_void_p,
                                              ctypes.c_void_p, ctypes.c_float, ctypes.c_int32, ctypes.c_void_p,
                                              ctypes.c_void_p]
    lib.wushkv_decode_attn_test_timeout.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(CacheBufs),
                                                    ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float,
                                                    ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                                    ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p]
    lib.wushkv_gram_accumulate.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p,
                                           ctypes.c_void_p]
    for name in SYMBOLS:
        getattr(lib, name).restype = ctypes.c_int
    return lib


lib = _load()


def _check(rc: int, what: str) -> None:
    if rc != OK:
        raise WushKVError(f"{what}: {_ERR.get(rc, rc)}")


def make_config(batch, n_kv_heads, n_q_heads, bits, capacity, s_sink, s_keep, s_flush=16, chunk_max=1,
                p_lo=1.0, p_hi=99.0, head_dim=128, transform=TRANSFORM_DENSE, quantizer=QUANT_PERCENTILE,
                clip_alpha=0.0) -> Config:
    return Config(batch, n_kv_heads, n_q_heads, head_dim, bits, capacity, s_sink, s_keep, s_flush, chunk_max,
                  p_lo, p_hi, transform, quantizer, clip_alpha)


def pack_layout(cfg: Config) -> Layout:
    out = Layout()
    _check(lib.wushkv_pack_layout(ctypes.byref(cfg), ctypes.byref(out)), "wushkv_pack_layout")
    return out


def compensation(t_k: torch.Tensor) -> torch.Tensor:
    """T_K^{-1} (fp32, host) of host fp16 T_K [H_kv, 128, 128] via the library's Gauss-Jordan."""
    t = t_k.detach().to("cpu", torch.float16).contiguous()
    out = torch.empty(t.shape, dtype=torch.float32)
    _check(lib.wushkv_compensation(t.data_ptr(), t.shape[0], out.data_ptr()), "wushkv_compensation")
    return out


def hadamard_compensation(n_kv_heads: int) -> torch.Tensor:
    """T_K^{-1} (fp32, host) of the in-kernel Hadamard transform: H itself (wushkv_hadamard)."""
    out = torch.empty(n_kv_heads, 128, 128, dtype=torch.float32)
    _check(lib.wushkv_hadamard(n_kv_heads, out.data_ptr()), "wushkv_hadamard")
    return out


def gram_accumulate(x: torch.Tensor, gram: torch.Tensor, stream=None) -> torch.Tensor:
    """gram[h] += sum_t x[t, h] x[t, h]^T on the device (wushkv_gram_accumulate).
    x: fp16 [..., n_heads, 128], contiguous (leading dimensions are tokens);
    gram: fp64 [n_heads, 128, 128], contiguous.  Returns gram."""
    if x.dtype != torch.float16 or gram.dtype != torch.float64 or not x.is_contiguous() \
            or not gram.is_contiguous() or x.dim() < 2 or x.shape[-1] != 128 \
            or tuple(gram.shape) != (x.shape[-2], 128, 128):
        raise WushKVError("gram_accumulate: x must be contiguous fp16 [..., H, 128], gram fp64 [H, 128, 128]")
    _require_cuda(x, gram)
    if x.device != gram.device:
        raise WushKVError("gram_accumulate: x and gram must be on the same device")
    n_heads = x.shape[-2]
    n_tokens = x.numel() // (n_heads * 128) if n_heads else 0
    _check(lib.wushkv_gram_accumulate(x.data_ptr(), n_tokens, n_heads, gram.data_ptr(), _stream_ptr(stream)),
           "wushkv_gram_accumulate")
    return gram


def _require_cuda(*tensors) -> None:
    """The library reads and writes these through device pointers: a host tensor would hand
    a kernel an address it cannot use, so it is refused here (None entries are skipped)."""
    for t in tensors:
        if t is not None and not t.is_cuda:
            raise WushKVError("expected CUDA tensors: the library's kernels read them on the device")


def _ptr(t: Optional[torch.Tensor]):
    return t.data_ptr() if t is not None else None


def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


class KVCache:
    """One layer's cache buffers, allocated with torch on `device` per the library's layout."""

    def __init__(self, cfg: Config, device="cuda"):
        self.cfg = cfg
        self.layout = pack_layout(cfg)
        L = self.layout
        u8 = dict(dtype=torch.uint8, device=device)
        self.k_codes = torch.zeros(L.codes_bytes, **u8)
        self.v_codes = torch.zeros(L.codes_bytes, **u8)
        self.k_params = torch.zeros(L.params_bytes // 4, dtype=torch.int32, device=device)
        self.v_params = torch.zeros(L.params_bytes // 4, dtype=torch.int32, device=device)
        self.k_sink = torch.zeros(L.sink_bytes // 2, dtype=torch.float16, device=device)
        self.v_sink = torch.zeros(L.sink_bytes // 2, dtype=torch.float16, device=device)
        self.k_ring = torch.zeros(L.ring_bytes // 2, dtype=torch.float16, device=device)
        self.v_ring = torch.zeros(L.ring_bytes // 2, dtype=torch.float16, device=device)
        self.state = torch.zeros(L.state_bytes // 4, dtype=torch.int32, device=device)
        # one scratch buffer serves decode_attn / step and chunk_attn (never concurrently)
        self.workspace = torch.zeros(max(L.workspace_bytes, L.chunk_workspace_bytes), **u8)
        self.bufs = CacheBufs(*(t.data_ptr() for t in (self.k_codes, self.v_codes, self.k_params, self.v_params,
                                                        self.k_sink, self.v_sink, self.k_ring, self.v_ring,
                                                        self.state)))

    @property
    def units(self) -> int:
        return self.cfg.batch * self.cfg.n_kv_heads

    def lengths(self):
        """(S, S_quant) per (sequence, KV head): int32 [B, H_kv] each (device tensors)."""
        st = self.state[: 2 * self.units].view(self.cfg.batch, self.cfg.n_kv_heads, 2)
        return st[..., 0], st[..., 1]

    def status(self) -> int:
        return int(self.state[2 * self.units].item())

    def reset(self) -> None:
        self.state.zero_()

    def append(self, k_new: torch.Tensor, v_new: torch.Tensor, t_k: torch.Tensor, stream=None) -> None:
        """k_new, v_new: fp16 [B, n_new, H_kv, 128] on the device; t_k fp16 [H_kv, 128, 128]."""
        _require_cuda(k_new, v_new, t_k)
        n_new = k_new.shape[1]
        _check(lib.wushkv_append(ctypes.byref(self.cfg), ctypes.byref(self.bufs), k_new.data_ptr(),
                                 v_new.data_ptr(), n_new, _ptr(t_k), _stream_ptr(stream)), "wushkv_append")

    def decode_attn(self, q: torch.Tensor, t_k_inv: torch.Tensor, softmax_scale: float,
                    out: Optional[torch.Tensor] = None, out_fp16: bool = False, stream=None) -> torch.Tensor:
        """q fp16 [B, H_q, 128]; t_k_inv fp32 [H_kv, 128, 128] (T_K^{-1}); returns out [B, H_q, 128]."""
        _require_cuda(q, t_k_inv, out)
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float16 if out_fp16 else torch.float32, device=q.device)
        _check(lib.wushkv_decode_attn(ctypes.byref(self.cfg), ctypes.byref(self.bufs), q.data_ptr(),
                                      t_k_inv.data_ptr(), float(softmax_scale), 1 if out.dtype == torch.float16 else 0,
                                      out.data_ptr(), self.workspace.data_ptr(), _stream_ptr(stream)),
               "wushkv_decode_attn")
        return out

    def chunk_attn(self, q: torch.Tensor, t_k_inv: torch.Tensor, softmax_scale: float,
                   out: Optional[torch.Tensor] = None, out_fp16: bool = False, stream=None) -> torch.Tensor:
        """q fp16 [B, n, H_q, 128]: the n newest positions' queries (the chunk just appended,
        n <= chunk_max), each attending causally over the cache; returns out [B, n, H_q, 128]."""
        _require_cuda(q, t_k_inv, out)
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float16 if out_fp16 else torch.float32, device=q.device)
        _check(lib.wushkv_chunk_attn(ctypes.byref(self.cfg), ctypes.byref(self.bufs), q.data_ptr(), q.shape[1],
                                     t_k_inv.data_ptr(), float(softmax_scale), 1 if out.dtype == torch.float16 else 0,
                                     out.data_ptr(), self.workspace.data_ptr(), _stream_ptr(stream)),
               "wushkv_chunk_attn")
        return out

    def step(self, k_new: torch.Tensor, v_new: torch.Tensor, t_k: torch.Tensor, q: torch.Tensor,
             t_k_inv: torch.Tensor, softmax_scale: float, out: Optional[torch.Tensor] = None,
             out_fp16: bool = False, stream=None) -> torch.Tensor:
        """append(k_new, v_new) then decode_attn(q) in one call (wushkv_step)."""
        _require_cuda(k_new, v_new, t_k, q, t_k_inv, out)
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float16 if out_fp16 else torch.float32, device=q.device)
        _check(lib.wushkv_step(ctypes.byref(self.cfg), ctypes.byref(self.bufs), k_new.data_ptr(), v_new.data_ptr(),
                               k_new.shape[1], _ptr(t_k), q.data_ptr(), t_k_inv.data_ptr(), float(softmax_scale),
                               1 if out.dtype == torch.float16 else 0, out.data_ptr(), self.workspace.data_ptr(),
                               _stream_ptr(stream)),
               "wushkv_step")
        return out

    def step_prep(self, k_raw: torch.Tensor, v_new: torch.Tensor, t_k: torch.Tensor, q_raw: torch.Tensor,
                  t_k_inv: torch.Tensor, softmax_scale: float, rope_theta: float,
                  q_norm_gain: Optional[torch.Tensor] = None, k_norm_gain: Optional[torch.Tensor] = None,
                  norm_eps: float = 1e-6, out: Optional[torch.Tensor] = None, out_fp16: bool = False,
                  stream=None) -> torch.Tensor:
        """step() on raw projections: per-head RMSNorm (gains given) and RoPE inside the
        library's kernels (wushkv_step_prep).  Gains: fp16 [128] on the device."""
        _require_cuda(k_raw, v_new, t_k, q_raw, t_k_inv, q_norm_gain, k_norm_gain, out)
        if out is None:
            out = torch.empty(q_raw.shape, dtype=torch.float16 if out_fp16 else torch.float32, device=q_raw.device)
        prep = Prep(float(rope_theta), q_norm_gain.data_ptr() if q_norm_gain is not None else None,
                    k_norm_gain.data_ptr() if k_norm_gain is not None else None, float(norm_eps))
        _check(lib.wushkv_step_prep(ctypes.byref(self.cfg), ctypes.byref(self.bufs), k_raw.data_ptr(),
                                    v_new.data_ptr(), k_raw.shape[1], _ptr(t_k), q_raw.data_ptr(),
                                    t_k_inv.data_ptr(), float(softmax_scale), 1 if out.dtype == torch.float16 else 0,
                                    out.data_ptr(), self.workspace.data_ptr(), ctypes.byref(prep),
                                    _stream_ptr(stream)),
               "wushkv_step_prep")
        return out

    def decode_attn_static(self, q: torch.Tensor, t_k_inv: torch.Tensor, softmax_scale: float,
                           out: torch.Tensor, stream=None) -> torch.Tensor:
        """decode_attn through wushkv_decode_attn_static: scratch in the library's own device
        array, `out` supplied by the caller (fp32 or fp16), nothing allocated."""
        _require_cuda(q, t_k_inv, out)
        _check(lib.wushkv_decode_attn_static(ctypes.byref(self.cfg), ctypes.byref(self.bufs), q.data_ptr(),
                                             t_k_inv.data_ptr(), float(softmax_scale),
                                             1 if out.dtype == torch.float16 else 0, out.data_ptr(),
                                             _stream_ptr(stream)),
               "wushkv_decode_attn_static")
        return out

    def decode_attn_test_timeout(self, q: torch.Tensor, t_k_inv: torch.Tensor, softmax_scale: float,
                                 out: torch.Tensor, withhold_stage: int, wait_limit_cycles: int,
                                 stream=None) -> torch.Tensor:
        """The bounded-wait test hook (wushkv_decode_attn_test_timeout): a shortened wait
        limit and one withheld pipeline stage per work item."""
        _require_cuda(q, t_k_inv, out)
        _check(lib.wushkv_decode_attn_test_timeout(ctypes.byref(self.cfg), ctypes.byref(self.bufs), q.data_ptr(),
                                                   t_k_inv.data_ptr(), float(softmax_scale),
                                                   1 if out.dtype == torch.float16 else 0, out.data_ptr(),
                                                   self.workspace.data_ptr(), int(withhold_stage),
                                                   int(wait_limit_cycles), _stream_ptr(stream)),
               "wushkv_decode_attn_test_timeout")
        return out

    # -- typed views of the buffers (for tests and tools) ------------------------
    def codes_view(self, kind: str) -> torch.Tensor:
        """uint8 [B, H_kv, cap_alloc, code_bytes]."""
        t = self.k_codes if kind == "k" else self.v_codes
        return t.view(self.cfg.batch, self.cfg.n_kv_heads, self.layout.cap_alloc, self.layout.code_bytes)

    def params_view(self, kind: str) -> torch.Tensor:
        """fp16 [B, H_kv, cap_alloc, 2] = (s, z)."""
        t = self.k_params if kind == "k" else self.v_params
        return t.view(torch.float16).view(self.cfg.batch, self.cfg.n_kv_heads, self.layout.cap_alloc, 2)

    def sink_view(self, kind: str) -> torch.Tensor:
        t = self.k_sink if kind == "k" else self.v_sink
        return t.view(self.cfg.batch, self.cfg.n_kv_heads, -1, 128)

    def ring_view(self, kind: str) -> torch.Tensor:
        t = self.k_ring if kind == "k" else self.v_ring
        return t.view(self.cfg.batch, self.cfg.n_kv_heads, self.layout.ring_slots, 128)


def config_for_workload(wl, extra_capacity: int = 1024, chunk_max: int = 1) -> Config:
    """Library config of a synthetic workload (synth.Workload); capacity = context + extra."""
    return make_config(wl.batch, wl.n_kv_heads, wl.n_q_heads, wl.bits, wl.context + extra_capacity,
                       wl.s_sink, wl.s_keep, wl.s_flush, chunk_max, wl.p_lo, wl.p_hi, wl.head_dim)
