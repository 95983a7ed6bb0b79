"""The in-kernel Walsh-Hadamard key transform (config transform = HADAMARD, no T_K
argument) against the oracle with T_K = H in float64, through the C ABI: small and bulk
appends within the general-transform bounds (the GPU sums the butterflies in fp32),
decode parity on the GPU's own cache with H as the compensation."""
import numpy as np
import pytest
import torch

from decode_attention_head_b200 import binding as bnd
from oracle import transform as otr
from tests import harness as H

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bits,Hkv,Hq,chunks", [
    (2, 2, 8, [1] * 40 + [500] + [1] * 30 + [300] + [1] * 9),
    (4, 2, 4, [700] + [1] * 50),
])
def test_hadamard_transform_matches_oracle(bits, Hkv, Hq, chunks):
    B = 2
    cfg = bnd.make_config(B, Hkv, Hq, bits, 2000, 4, 32, 16, 1, transform=bnd.TRANSFORM_HADAMARD)
    rng = np.random.default_rng(bits + Hq)
    T = np.broadcast_to(otr.hadamard(128), (Hkv, 128, 128)).copy()   # float64, exact H
    tinv = bnd.hadamard_compensation(Hkv).cuda()
    gc = bnd.KVCache(cfg)
    oc = H.oracle_cache_for(cfg)
    scale = 1 / np.sqrt(128)
    for i, n in enumerate(chunks):
        k = rng.standard_normal((B, n, Hkv, 128))
        k[..., [7, 70]] *= 20  # outlier channels, spread by the rotation
        k = k.astype(np.float16)
        v = rng.standard_normal((B, n, Hkv, 128)).astype(np.float16)
        gc.append(H.to_dev(k), H.to_dev(v), None)
        oc.append(k, v, T)
        if i % 10 == 0 or n > 1:
            q = rng.standard_normal((B, Hq, 128)).astype(np.float16)
            out = gc.decode_attn(H.to_dev(q), tinv, scale)
            torch.cuda.synchronize()
            ref = H.oracle_decode(H.oracle_cache_from_gpu(gc), q, T, scale)
            H.assert_attention_close(out.cpu().numpy(), ref)
    torch.cuda.synchronize()
    assert gc.status() == 0
    st = H.compare_caches(oc, H.download(gc), cfg, gc.layout.ring_slots, exact=False)
    print(f"[hadamard] cache vs oracle: {st}")
    assert st["code_maxdiff"] <= 1 and st["code_diff"] <= 1e-4 * st["code_elems"], st
    assert st["fp16_maxulp"] <= 8 and st["fp16_diff"] <= 2e-3 * st["fp16_elems"], st
    assert st["param_diff"] <= 0.02 * st["param_tokens"], st
