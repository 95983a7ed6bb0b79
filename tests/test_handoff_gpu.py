"""The exact append handoff under a general T_K.

With a random (non-identity) key transform the GPU accumulates k' = T_K k in fp32 and the
oracle in double, so a k' next to an fp16 rounding midpoint may round differently and the
whole-path comparison in test_append_gpu.py can only bound the differences.  The
quantizer itself must still be exact: this test feeds the oracle's quantizer the GPU's own
fp16 k' and requires the GPU's codes and (s, z) bit for bit ("WUSH-KV: KV Cache
Quantization with Data-Adaptive Transforms", §5.3, the percentile-clipped affine quantizer;
§4.3 / Appendix B.3 for the RMS-scaled grid).

* Flush path: chunks of n <= chunk_max tokens stay fp16 in the ring until the next append
  flushes them; the ring rows are read back before that append and quantized by the oracle.
* Bulk path (n > chunk_max quantizes straight from the transform's registers): a second
  cache with a recent window wider than the chunk keeps every transformed row fp16; the
  transform of a row does not depend on its route, so those rows are the first cache's
  quantizer inputs.
"""
import numpy as np
import pytest
import torch

from decode_attention_head_b200 import binding as bnd
from decode_attention_head_b200 import synth
from oracle import quantizer as oq
from oracle import quest as oqt
from tests import harness as H

pytestmark = pytest.mark.gpu


def _tokens(rng, B, n, Hkv, outliers=True):
    x = rng.standard_normal((B, n, Hkv, 128))
    if outliers:
        x[..., [5, 40, 77, 119]] *= 20
    return x.astype(np.float16)


def _quantizer(cfg, rms_alpha):
    if rms_alpha is None:
        return lambda x: oq.quantize(x, cfg.bits, cfg.p_lo, cfg.p_hi)
    return lambda x: oqt.quantize(x, cfg.bits, rms_alpha)


def _check_rows(g, b, h, kind, pos, rows, qfn):
    c, s, z = qfn(rows)
    np.testing.assert_array_equal(g[f"{kind}_codes"][b, h, pos], c)
    np.testing.assert_array_equal(g[f"{kind}_s"][b, h, pos].view(np.uint16), s.view(np.uint16))
    np.testing.assert_array_equal(g[f"{kind}_z"][b, h, pos].view(np.uint16), z.view(np.uint16))


@pytest.mark.parametrize("bits,rms", [(2, False), (4, False), (2, True)])
def test_flush_quantizes_the_gpu_fp16_rows_exactly(bits, rms):
    alpha = oqt.gaussian_optimal_alpha(bits) if rms else None
    extra = {"quantizer": bnd.QUANT_RMS, "clip_alpha": alpha} if rms else {}
    cfg = bnd.make_config(2, 2, 8, bits, 1500, 4, 32, 16, 48, **extra)
    wl = synth.WORKLOADS["tiny"]
    T = np.stack([synth.key_transform(wl, 3, h).numpy() for h in range(2)])
    t_dev = H.to_dev(T)
    qfn = _quantizer(cfg, alpha)
    rng = np.random.default_rng(40 + bits + 7 * rms)
    gc = bnd.KVCache(cfg)
    R = gc.layout.ring_slots
    checked = 0
    for n in [48, 17, 48, 1, 33, 48, 5, 48, 48, 2]:
        before = H.download(gc)
        gc.append(H.to_dev(_tokens(rng, 2, n, 2)), H.to_dev(_tokens(rng, 2, n, 2, False)), t_dev)
        torch.cuda.synchronize()
        after = H.download(gc)
        assert after["status"] == 0
        for b in range(2):
            for h in range(2):
                lo, hi = int(before["Sq"][b, h]), int(after["Sq"][b, h])
                lo = max(lo, cfg.s_sink)
                if hi <= lo:
                    continue
                pos = np.arange(lo, hi)
                for kind in ("k", "v"):
                    rows = before[f"{kind}_ring"][b, h][pos % R]
                    _check_rows(after, b, h, kind, pos, rows, qfn)
                checked += len(pos)
    assert checked >= 200


@pytest.mark.parametrize("bits", [2, 4])
def test_bulk_quantizes_the_gpu_transform_exactly(bits):
    n0, n = 37, 900
    cfg_q = bnd.make_config(1, 2, 4, bits, 1100, 4, 32, 16, 1)
    cfg_k = bnd.make_config(1, 2, 4, bits, 1100, 4, 1024, 16, 1)
    wl = synth.WORKLOADS["tiny"]
    T = np.stack([synth.key_transform(wl, 5, h).numpy() for h in range(2)])
    t_dev = H.to_dev(T)
    rng = np.random.default_rng(60 + bits)
    k0, v0 = _tokens(rng, 1, n0, 2), _tokens(rng, 1, n0, 2, False)
    k1, v1 = _tokens(rng, 1, n, 2), _tokens(rng, 1, n, 2, False)
    caches = []
    for cfg in (cfg_q, cfg_k):
        gc = bnd.KVCache(cfg)
        gc.append(H.to_dev(k0), H.to_dev(v0), t_dev)   # an unaligned start for the bulk chunk
        gc.append(H.to_dev(k1), H.to_dev(v1), t_dev)
        caches.append(gc)
    torch.cuda.synchronize()
    gq, gk = H.download(caches[0]), H.download(caches[1])
    assert gq["status"] == 0 and gk["status"] == 0
    assert int(gk["Sq"][0, 0]) == 0  # the wide window kept every row fp16
    Rk = caches[1].layout.ring_slots
    qfn = _quantizer(cfg_q, None)
    for h in range(2):
        lo, hi = cfg_q.s_sink, int(gq["Sq"][0, h])
        assert hi > n0 + 500
        pos = np.arange(lo, hi)
        _check_rows(gq, 0, h, "k", pos, gk["k_ring"][0, h][pos % Rk], qfn)
        _check_rows(gq, 0, h, "v", pos, gk["v_ring"][0, h][pos % Rk], qfn)
