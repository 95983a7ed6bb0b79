"""Shared helpers of the GPU parity tests: build oracle caches, upload them into the
library's buffers (documented layout), read GPU caches back, and compare.

Test infrastructure: it imports the oracle and the binding, never the reverse.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import attention as oatt
from oracle import cache as ocache
from oracle import quantizer as oq

# attention-output tolerance of the path's specification (2e-3 max abs, 1e-3 relative): both must hold,
# the relative one on the 2-norm of each output row
ATOL = 2e-3
RTOL = 1e-3


def _vgroup_index(bits):
    """[16, 8*bits]: the 16-bit half of a 16-position value group that holds chunk c (bytes
    2c, 2c+1 of the row's packed record) of group position r (the value layout of wushkv.h)."""
    nc = 8 * bits
    idx = np.empty((16, nc), np.int64)
    for r in range(16):
        t = r & 7
        for c in range(nc):
            lp = 4 * (t & 3) + 2 * (c & 1) + (t >> 2)
            w = 16 * (c >> 1) + lp if bits == 2 else 128 * ((c >> 1) & 1) + 16 * (c >> 2) + lp
            idx[r, c] = 2 * w + (r >> 3)
    return idx


def v_rows_from_groups(buf: np.ndarray, bits: int) -> np.ndarray:
    """Value codes as stored (uint8 [..., positions, 16*bits], positions a multiple of 16) ->
    one packed record per position, the key layout."""
    buf = np.ascontiguousarray(buf)
    shp = buf.shape
    halves = buf.reshape(shp[:-2] + (shp[-2] // 16, 16 * shp[-1])).view(np.uint16)
    rows = halves[..., _vgroup_index(bits)]
    return np.ascontiguousarray(rows).reshape(shp[:-2] + (shp[-2], shp[-1] // 2)).view(np.uint8)


def v_groups_from_rows(rows: np.ndarray, bits: int) -> np.ndarray:
    """Inverse of v_rows_from_groups."""
    rows = np.ascontiguousarray(rows)
    shp = rows.shape
    r16 = rows.view(np.uint16).reshape(shp[:-2] + (shp[-2] // 16, 16, shp[-1] // 2))
    out = np.zeros(shp[:-2] + (shp[-2] // 16, 8 * shp[-1]), np.uint16)
    out[..., _vgroup_index(bits)] = r16
    return out.view(np.uint8).reshape(shp)


def stored_codes(gc, kind, b=None, h=None) -> np.ndarray:
    """One packed record per position of the GPU cache's codes (uint8 [..., cap_alloc, CB])."""
    t = gc.codes_view(kind) if b is None else gc.codes_view(kind)[b, h]
    a = t.cpu().numpy()
    return v_rows_from_groups(a, gc.cfg.bits) if kind == "v" else a


def oracle_cache_for(cfg, store_dtype=np.float16) -> ocache.Cache:
    return ocache.Cache(cfg.batch, cfg.n_kv_heads, 128, cfg.bits, cfg.p_lo, cfg.p_hi, cfg.s_sink, cfg.s_keep,
                        cfg.s_flush, capacity=cfg.capacity, chunk_max=cfg.chunk_max, store_dtype=store_dtype)


def upload(oc: ocache.Cache, gc) -> None:
    """Write the oracle cache's contents into the GPU cache buffers (layout of wushkv.h)."""
    cfg, L = gc.cfg, gc.layout
    B, H = cfg.batch, cfg.n_kv_heads
    cap = min(oc.capacity, L.cap_alloc)
    assert int(oc.S.max()) <= cap
    for kind in ("k", "v"):
        codes = getattr(oc, f"{kind}_codes")[:, :, :cap]
        packed = np.zeros((B, H, L.cap_alloc, L.code_bytes), dtype=np.uint8)
        packed[:, :, :cap] = oq.pack(codes, cfg.bits)
        if kind == "v":
            packed = v_groups_from_rows(packed, cfg.bits)
        gc.codes_view(kind).copy_(torch.from_numpy(packed))
        s = getattr(oc, f"{kind}_s")
        z = getattr(oc, f"{kind}_z")
        par = np.zeros((B, H, L.cap_alloc, 2), dtype=np.float16)
        par[:, :, :cap, 0] = s[:, :, :cap]
        par[:, :, :cap, 1] = z[:, :, :cap]
        gc.params_view(kind).copy_(torch.from_numpy(par))
        store = getattr(oc, f"{kind}_store")
        sink = np.zeros(tuple(gc.sink_view(kind).shape), dtype=np.float16)
        ring = np.zeros(tuple(gc.ring_view(kind).shape), dtype=np.float16)
        for b in range(B):
            S, Sq = int(oc.S[b]), int(oc.S_quant[b])
            ns = min(cfg.s_sink, S)
            sink[b, :, :ns] = store[b, :, :ns]
            for p in range(max(Sq, cfg.s_sink), S):
                ring[b, :, p % L.ring_slots] = store[b, :, p]
        gc.sink_view(kind).copy_(torch.from_numpy(sink))
        gc.ring_view(kind).copy_(torch.from_numpy(ring))
    st = np.zeros(gc.state.numel(), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            st[2 * (b * H + h)] = oc.S[b]
            st[2 * (b * H + h) + 1] = oc.S_quant[b]
    gc.state.copy_(torch.from_numpy(st))


def download(gc):
    """GPU cache contents as numpy: dict with S, Sq [B,H], codes/params per kind, sink, ring."""
    S, Sq = (t.cpu().numpy() for t in gc.lengths())
    out = {"S": S, "Sq": Sq, "status": gc.status()}
    for kind in ("k", "v"):
        out[f"{kind}_codes"] = oq.unpack(stored_codes(gc, kind), gc.cfg.bits)
        par = gc.params_view(kind).cpu().numpy()
        out[f"{kind}_s"] = par[..., 0]
        out[f"{kind}_z"] = par[..., 1]
        out[f"{kind}_sink"] = gc.sink_view(kind).cpu().numpy()
        out[f"{kind}_ring"] = gc.ring_view(kind).cpu().numpy()
    return out


def compare_caches(oc: ocache.Cache, g, cfg, ring_slots, exact=True, kinds=("k", "v")):
    """Compare a downloaded GPU cache with the oracle.  exact=True: bit-exact everywhere.
    exact=False: returns mismatch statistics for the caller to bound."""
    B, H = cfg.batch, cfg.n_kv_heads
    stats = {"code_elems": 0, "code_diff": 0, "code_maxdiff": 0, "param_tokens": 0, "param_diff": 0,
             "fp16_elems": 0, "fp16_diff": 0, "fp16_maxulp": 0}
    for b in range(B):
        S, Sq = int(oc.S[b]), int(oc.S_quant[b])
        assert (g["S"][b] == S).all(), (b, g["S"][b], S)
        assert (g["Sq"][b] == Sq).all(), (b, g["Sq"][b], Sq)
        qpos = np.arange(cfg.s_sink, Sq) if Sq > cfg.s_sink else np.arange(0)
        for kind in kinds:
            oc_codes = getattr(oc, f"{kind}_codes")[b][:, qpos]
            gc_codes = g[f"{kind}_codes"][b][:, qpos]
            d = np.abs(oc_codes.astype(np.int32) - gc_codes.astype(np.int32))
            stats["code_elems"] += d.size
            stats["code_diff"] += int((d != 0).sum())
            stats["code_maxdiff"] = max(stats["code_maxdiff"], int(d.max()) if d.size else 0)
            for nm in ("s", "z"):
                o = getattr(oc, f"{kind}_{nm}")[b][:, qpos]
                gv = g[f"{kind}_{nm}"][b][:, qpos]
                pd = o.view(np.uint16) != gv.view(np.uint16)
                stats["param_tokens"] += pd.size
                stats["param_diff"] += int(pd.sum())
            store = getattr(oc, f"{kind}_store")[b].astype(np.float16)
            ns = min(cfg.s_sink, S)
            fp_o = [store[:, :ns]]
            fp_g = [g[f"{kind}_sink"][b][:, :ns]]
            rpos = np.arange(max(Sq, cfg.s_sink), S)
            fp_o.append(store[:, rpos])
            fp_g.append(g[f"{kind}_ring"][b][:, rpos % ring_slots])
            fo = np.concatenate(fp_o, axis=1).view(np.int16).astype(np.int32)
            fg = np.concatenate(fp_g, axis=1).view(np.int16).astype(np.int32)
            ud = np.abs(fo - fg)
            stats["fp16_elems"] += ud.size
            stats["fp16_diff"] += int((ud != 0).sum())
            stats["fp16_maxulp"] = max(stats["fp16_maxulp"], int(ud.max()) if ud.size else 0)
    if exact:
        assert stats["code_diff"] == 0, stats
        assert stats["param_diff"] == 0, stats
        assert stats["fp16_diff"] == 0, stats
    return stats


def assert_attention_close(gpu: np.ndarray, ref: np.ndarray, atol=ATOL, rtol=RTOL):
    gpu = np.asarray(gpu, dtype=np.float64)
    err = np.abs(gpu - ref)
    assert np.isfinite(gpu).all()
    assert err.max() <= atol, f"max abs err {err.max():.3e}"
    num = np.linalg.norm((gpu - ref).reshape(-1, ref.shape[-1]), axis=-1)
    den = np.linalg.norm(ref.reshape(-1, ref.shape[-1]), axis=-1)
    rel = num / np.maximum(den, 1e-30)
    print(f"[parity] max_abs={err.max():.3e} max_row_rel={rel.max():.3e}")
    assert rel.max() <= rtol, f"max row-relative err {rel.max():.3e}"
    return float(err.max()), float(rel.max())


def oracle_cache_from_gpu(gc) -> ocache.Cache:
    """An oracle cache holding exactly the GPU cache's contents (state, codes, (s, z), fp16
    windows), so that decode parity is measured on an identical cache."""
    cfg, L = gc.cfg, gc.layout
    g = download(gc)
    oc = ocache.Cache(cfg.batch, cfg.n_kv_heads, 128, cfg.bits, cfg.p_lo, cfg.p_hi, cfg.s_sink, cfg.s_keep,
                      cfg.s_flush, capacity=L.cap_alloc, chunk_max=cfg.chunk_max)
    for b in range(cfg.batch):
        S, Sq = int(g["S"][b].max()), int(g["Sq"][b].max())
        assert (g["S"][b] == S).all() and (g["Sq"][b] == Sq).all()
        oc.S[b], oc.S_quant[b] = S, Sq
        for kind in ("k", "v"):
            getattr(oc, f"{kind}_codes")[b] = g[f"{kind}_codes"][b]
            getattr(oc, f"{kind}_s")[b] = g[f"{kind}_s"][b]
            getattr(oc, f"{kind}_z")[b] = g[f"{kind}_z"][b]
            store = getattr(oc, f"{kind}_store")
            ns = min(cfg.s_sink, S)
            store[b, :, :ns] = g[f"{kind}_sink"][b][:, :ns]
            rpos = np.arange(max(Sq, cfg.s_sink), S)
            store[b][:, rpos] = g[f"{kind}_ring"][b][:, rpos % L.ring_slots]
    return oc


def oracle_decode(oc, q_np, T_K_np, scale):
    return oatt.decode(oc, q_np, T_K_np, scale)


def to_dev(x: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to(device)
