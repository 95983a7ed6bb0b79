"""The RMS-scaled symmetric (QuEST-style) quantizer on the GPU (config quantizer = RMS)
against the oracle's (oracle/quest.py), through the C ABI: with an identity T_K every code,
(s, z) and fp16 window value is bit-exact across decode-style and bulk appends at 2 and 4
bits; decode attention over the cache matches the oracle within the tolerance."""
import numpy as np
import pytest
import torch

from decode_attention_head_b200 import binding as bnd
from oracle import cache as ocache
from oracle import quest as oqt
from tests import harness as H

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bits", [2, 4])
def test_rms_quantizer_bit_exact(bits):
    alpha = float(np.float32(oqt.gaussian_optimal_alpha(bits)))
    cfg = bnd.make_config(2, 2, 8, bits, 2000, 4, 32, 16, 1, quantizer=bnd.QUANT_RMS, clip_alpha=alpha)
    T = np.broadcast_to(np.eye(128, dtype=np.float16), (2, 128, 128)).copy()
    oc = ocache.Cache(2, 2, 128, bits, 1.0, 99.0, 4, 32, 16, capacity=2000, chunk_max=1,
                      quantize_fn=lambda x: oqt.quantize(x, bits, alpha))
    gc = bnd.KVCache(cfg)
    rng = np.random.default_rng(bits)
    t_dev = H.to_dev(T)
    for n in [1] * 40 + [600] + [1] * 30 + [333] + [1] * 5:
        k = rng.standard_normal((2, n, 2, 128))
        k[..., [3, 77]] *= 25
        k = k.astype(np.float16)
        v = (rng.standard_normal((2, n, 2, 128)) * rng.uniform(0.1, 10, (2, n, 2, 1))).astype(np.float16)
        oc.append(k, v, T)
        gc.append(H.to_dev(k), H.to_dev(v), t_dev)
    torch.cuda.synchronize()
    g = H.download(gc)
    assert g["status"] == 0
    H.compare_caches(oc, g, cfg, gc.layout.ring_slots, exact=True)
    q = rng.standard_normal((2, 8, 128)).astype(np.float16)
    tinv = bnd.compensation(torch.from_numpy(T)).cuda()
    out = gc.decode_attn(H.to_dev(q), tinv, 1 / np.sqrt(128))
    torch.cuda.synchronize()
    H.assert_attention_close(out.cpu().numpy(), H.oracle_decode(oc, q, T, 1 / np.sqrt(128)))
