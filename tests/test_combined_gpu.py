"""Every option of the path at once, through the C ABI: raw projections (wushkv_step_prep:
per-head RMSNorm + RoPE in the kernels), the in-kernel Walsh-Hadamard key transform and
the RMS-scaled symmetric (QuEST-style) quantizer, with decode steps of several tokens
(chunk_max 4) and bulk prefill chunks in between, fp16 output.  The oracle prepares the
same raw inputs (oracle/rope.py), transforms with H in float64 and quantizes with
oracle/quest.py; the cache must agree within the general-transform bounds and every
output must match exact attention over the GPU's own cache."""
import numpy as np
import pytest
import torch

from decode_attention_head_b200 import binding as bnd
from oracle import cache as ocache
from oracle import quest as oqt
from oracle import rope as orope
from oracle import transform as otr
from tests import harness as H

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bits,Hkv,Hq", [(2, 2, 8), (4, 1, 4)])
def test_all_options_together(bits, Hkv, Hq):
    B, theta, eps = 2, 1e6, 1e-6
    alpha = float(np.float32(oqt.gaussian_optimal_alpha(bits)))
    cfg = bnd.make_config(B, Hkv, Hq, bits, 3000, 4, 32, 16, 4, transform=bnd.TRANSFORM_HADAMARD,
                          quantizer=bnd.QUANT_RMS, clip_alpha=alpha)
    rng = np.random.default_rng(bits * 13 + Hq)
    T = np.broadcast_to(otr.hadamard(128), (Hkv, 128, 128)).copy()
    tinv = bnd.hadamard_compensation(Hkv).cuda()
    qg = rng.uniform(0.5, 1.5, 128).astype(np.float16)
    kg = rng.uniform(0.5, 1.5, 128).astype(np.float16)
    scale = 1 / np.sqrt(128)
    gc = bnd.KVCache(cfg)
    oc = ocache.Cache(B, Hkv, 128, bits, 1.0, 99.0, 4, 32, 16, capacity=3000, chunk_max=4,
                      quantize_fn=lambda x: oqt.quantize(x, bits, alpha))
    S = 0
    for i, n in enumerate([1] * 20 + [4, 3, 2] + [400] + [1] * 20 + [4] * 5 + [600] + [1] * 10):
        k_raw = (rng.standard_normal((B, n, Hkv, 128)) * 3).astype(np.float16)
        k_raw[..., [5, 99]] *= 8
        v = (rng.standard_normal((B, n, Hkv, 128)) * rng.uniform(0.2, 5, (B, n, Hkv, 1))).astype(np.float16)
        q_raw = (rng.standard_normal((B, Hq, 128)) * 3).astype(np.float16)
        out = gc.step_prep(H.to_dev(k_raw), H.to_dev(v), None, H.to_dev(q_raw), tinv, scale, theta,
                           H.to_dev(qg), H.to_dev(kg), eps, out_fp16=True)
        pos = (S + np.arange(n))[None, :, None]
        oc.append(orope.prepare(k_raw, pos, theta, kg, eps, True), v, T)
        q_rope = orope.prepare(q_raw, S + n - 1, theta, qg, eps, True)
        S += n
        torch.cuda.synchronize()
        assert gc.status() == 0
        assert out.dtype == torch.float16 and torch.isfinite(out).all()
        if i % 6 == 0 or n > 4:
            ref = H.oracle_decode(H.oracle_cache_from_gpu(gc), q_rope, T, scale)
            # fp16 output: one more rounding of the result
            H.assert_attention_close(out.float().cpu().numpy(), ref, atol=2e-3 + 1e-3 * np.abs(ref).max())
    assert np.array_equal(gc.lengths()[0][:, 0].cpu().numpy(), np.full(B, S))
    g = H.download(gc)
    st = H.compare_caches(oc, g, cfg, gc.layout.ring_slots, exact=False)
    print(f"[combined] cache vs oracle: {st}")
    assert st["code_maxdiff"] <= 1 and st["code_diff"] <= 1e-4 * st["code_elems"], st
    assert st["param_diff"] <= 0.02 * st["param_tokens"], st
    # fp16 window keys: the GPU sums the butterflies in fp32, the oracle in float64, so a key
    # may round to a neighbouring fp16 value; a key near zero (cancellation in the sum) is
    # off by more of its own ulps, so the error is measured in ulps of its row's magnitude
    worst = 0.0
    for b in range(B):
        Sq = int(g["Sq"][b, 0])
        ns = min(cfg.s_sink, S)
        rpos = np.arange(max(Sq, cfg.s_sink), S)
        gk = np.concatenate([g["k_sink"][b][:, :ns], g["k_ring"][b][:, rpos % gc.layout.ring_slots]], axis=1)
        ok = np.concatenate([oc.k_store[b][:, :ns], oc.k_store[b][:, rpos]], axis=1).astype(np.float64)
        rowmax = np.abs(ok).max(axis=-1, keepdims=True)
        ulp_row = np.exp2(np.floor(np.log2(np.maximum(rowmax, 2.0 ** -14))) - 10)
        worst = max(worst, float((np.abs(gk.astype(np.float64) - ok) / ulp_row).max()))
    print(f"[combined] fp16 window keys: max error {worst:.3f} ulps of the row magnitude")
    assert worst <= 1.0
