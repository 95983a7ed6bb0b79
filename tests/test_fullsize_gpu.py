"""Full-size parity: every model-shaped workload at its full size, in the launch
configuration the benchmark uses, checked on sampled (sequence, KV head) units.

The cache is filled on the GPU the way bench.py fills it (bulk appends of seeded synthetic
chunks, then a decode-style one-token append, or the prefill chunk for the prefill
workload). For each sampled unit:
  * append: the oracle replays the same chunks for that unit alone, and its cache is
    compared with the GPU's (values bit-exact; keys within the general-transform bound:
    codes off by at most 1 on at most 1e-4 of elements, k' within 8 fp16 ulps);
  * decode: the oracle attends over the GPU's own cache of that unit (downloaded through
    the documented layout), so decode error is measured on an identical cache, and the
    unit's query heads are compared within 2e-3 max abs / 1e-3 relative.
"""
import numpy as np
import pytest
import torch

import bench
from decode_attention_head_b200 import binding as bnd
from decode_attention_head_b200 import synth
from oracle import attention as oatt
from oracle import cache as ocache
from oracle import quantizer as oq
from tests import harness as H

pytestmark = pytest.mark.gpu


def _samples(wl):
    B, Hk = wl.batch, wl.n_kv_heads
    return sorted({(0, 0), (B // 2, Hk // 3), (B - 1, Hk - 1)})


def _unit_cache_from_gpu(gc, b, h, T):
    """An oracle Cache (one sequence, one KV head) holding the GPU cache of unit (b, h)."""
    cfg, L = gc.cfg, gc.layout
    S, Sq = (int(t[b, h].item()) for t in gc.lengths())
    oc = ocache.Cache(1, 1, 128, cfg.bits, cfg.p_lo, cfg.p_hi, cfg.s_sink, cfg.s_keep, cfg.s_flush,
                      capacity=L.cap_alloc, chunk_max=cfg.chunk_max)
    oc.S[0], oc.S_quant[0] = S, Sq
    for kind in ("k", "v"):
        codes = oq.unpack(H.stored_codes(gc, kind, b, h), cfg.bits)
        par = gc.params_view(kind)[b, h].cpu().numpy()
        getattr(oc, f"{kind}_codes")[0, 0] = codes
        getattr(oc, f"{kind}_s")[0, 0] = par[:, 0]
        getattr(oc, f"{kind}_z")[0, 0] = par[:, 1]
        store = getattr(oc, f"{kind}_store")
        ns = min(cfg.s_sink, S)
        store[0, 0, :ns] = gc.sink_view(kind)[b, h, :ns].cpu().numpy()
        rpos = np.arange(max(Sq, cfg.s_sink), S)
        store[0, 0, rpos] = gc.ring_view(kind)[b, h].cpu().numpy()[rpos % L.ring_slots]
    return oc


def _check_append(oc, gu, cfg):
    """Oracle unit cache `oc` vs the GPU unit cache `gu` (both one sequence, one head)."""
    S, Sq = int(oc.S[0]), int(oc.S_quant[0])
    assert (int(gu.S[0]), int(gu.S_quant[0])) == (S, Sq)
    q = np.arange(cfg.s_sink, Sq)
    w = np.concatenate([np.arange(min(cfg.s_sink, S)), np.arange(max(Sq, cfg.s_sink), S)])
    stats = {}
    for kind in ("k", "v"):
        c_o = getattr(oc, f"{kind}_codes")[0, 0, q].astype(np.int32)
        c_g = getattr(gu, f"{kind}_codes")[0, 0, q].astype(np.int32)
        d = np.abs(c_o - c_g)
        f_o = getattr(oc, f"{kind}_store")[0, 0, w].view(np.int16).astype(np.int32)
        f_g = getattr(gu, f"{kind}_store")[0, 0, w].view(np.int16).astype(np.int32)
        pdiff = sum(int((getattr(oc, f"{kind}_{nm}")[0, 0, q].view(np.uint16) !=
                         getattr(gu, f"{kind}_{nm}")[0, 0, q].view(np.uint16)).sum()) for nm in ("s", "z"))
        stats[kind] = dict(code_max=int(d.max()) if d.size else 0, code_diff=int((d != 0).sum()), n=d.size,
                           ulp_max=int(np.abs(f_o - f_g).max()) if f_o.size else 0, param_diff=pdiff,
                           tokens=len(q))
    print(f"[fullsize-append] {stats}")
    v, k = stats["v"], stats["k"]
    assert v["code_diff"] == 0 and v["param_diff"] == 0 and v["ulp_max"] == 0, v
    assert k["code_max"] <= 1 and k["code_diff"] <= 1e-4 * k["n"], k
    assert k["ulp_max"] <= 8, k
    assert k["param_diff"] <= 0.02 * 2 * k["tokens"], k


@pytest.mark.parametrize("name", ["llama3-8b-layer", "qwen3-8b-layer", "mha-32l", "prefill-append-decode"])
def test_full_size_workload_sampled_units(name):
    wl = synth.WORKLOADS[name]
    dev = torch.device("cuda")
    cfg = bench.layer_config(wl, bnd)
    layer = 0
    T = synth.key_transforms(wl, layer)
    tk, tinv = T.to(dev), bnd.compensation(T).to(dev)
    gc = bnd.KVCache(cfg, device=dev)
    units = _samples(wl)
    oracles = {u: ocache.Cache(1, 1, 128, cfg.bits, cfg.p_lo, cfg.p_hi, cfg.s_sink, cfg.s_keep, cfg.s_flush,
                               capacity=cfg.capacity, chunk_max=cfg.chunk_max) for u in units}
    Tn = T.numpy()

    def append(s0, n):
        kk = synth.bulk_tokens(wl, layer, s0, n, device=dev, which="k")
        vv = synth.bulk_tokens(wl, layer, s0, n, device=dev, which="v")
        gc.append(kk, vv, tk)
        for (b, h), oc in oracles.items():
            oc.append(kk[b:b + 1, :, h:h + 1].cpu().numpy(), vv[b:b + 1, :, h:h + 1].cpu().numpy(), Tn[h:h + 1])

    chunk = 4096 if wl.batch * wl.n_kv_heads <= 64 else 512
    if wl.prefill_chunk:
        base = wl.context - wl.prefill_chunk
        for s0 in range(0, base, chunk):
            append(s0, min(chunk, base - s0))
        append(base, wl.prefill_chunk)               # the prefill chunk: one bulk append
    else:
        for s0 in range(0, wl.context - 1, chunk):
            append(s0, min(chunk, wl.context - 1 - s0))
        append(wl.context - 1, 1)                    # decode-style append (deferred flush)
    q = synth.bulk_queries(wl, layer, wl.context, device=dev)
    out = gc.decode_attn(q, tinv, synth.default_softmax_scale(wl.head_dim))
    torch.cuda.synchronize()
    assert gc.status() == 0
    S, Sq = (t.cpu().numpy() for t in gc.lengths())
    assert (S == wl.context).all()
    assert (Sq > wl.context - wl.s_keep - wl.s_flush - 1).all()

    g = wl.group
    for (b, h), oc in oracles.items():
        gu = _unit_cache_from_gpu(gc, b, h, Tn[h])
        _check_append(oc, gu, cfg)
        ref = oatt.decode(gu, q[b:b + 1, h * g:(h + 1) * g].cpu().numpy(), Tn[h:h + 1],
                          synth.default_softmax_scale(wl.head_dim))[0]
        H.assert_attention_close(out[b, h * g:(h + 1) * g].cpu().numpy(), ref)


def test_full_size_chunk_attention_sampled_units():
    """Chunked prefill at the Llama-3-8B layer's full size, in the launch configuration the
    benchmark times: an 8-token chunk appended (decode-time path) onto 32,760 cached
    positions, its 8 queries attending causally in one launch pair (4 blocks of 2 tokens side
    by side).  Each sampled unit's 8 x 4 query rows are checked against the oracle's causal
    chunk attention over the GPU's own cache of that unit."""
    wl = synth.WORKLOADS["llama3-8b-layer"]
    n = 8
    dev = torch.device("cuda")
    cfg = bnd.config_for_workload(wl, extra_capacity=64, chunk_max=n)
    T = synth.key_transforms(wl, 0)
    tk, tinv = T.to(dev), bnd.compensation(T).to(dev)
    gc = bnd.KVCache(cfg, device=dev)
    base = wl.context - n
    for s0 in range(0, base, 4096):
        m = min(4096, base - s0)
        gc.append(synth.bulk_tokens(wl, 0, s0, m, device=dev, which="k"),
                  synth.bulk_tokens(wl, 0, s0, m, device=dev, which="v"), tk)
    gc.append(synth.bulk_tokens(wl, 0, base, n, device=dev, which="k"),
              synth.bulk_tokens(wl, 0, base, n, device=dev, which="v"), tk)
    q = torch.stack([synth.bulk_queries(wl, 0, base + t, device=dev) for t in range(n)], dim=1).contiguous()
    scale = synth.default_softmax_scale(wl.head_dim)
    out = gc.chunk_attn(q, tinv, scale)
    torch.cuda.synchronize()
    assert gc.status() == 0
    assert (gc.lengths()[0] == wl.context).all()
    Tn = T.numpy()
    g = wl.group
    for b, h in _samples(wl):
        gu = _unit_cache_from_gpu(gc, b, h, Tn[h])
        ref = oatt.chunk_decode(gu, q[b:b + 1, :, h * g:(h + 1) * g].cpu().numpy(), Tn[h:h + 1], scale)[0]
        H.assert_attention_close(out[b, :, h * g:(h + 1) * g].cpu().numpy(), ref)
