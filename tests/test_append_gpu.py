"""GPU append vs the oracle, through the C ABI.

Identity T_K: everything (state, codes, (s, z), fp16 windows) bit-exact.
Random T_K: k' = fp16(T_K k) is accumulated in fp32 on the GPU and in double in the
oracle, so k' may differ by one fp16 ulp next to a rounding midpoint; the accepted bound:
codes differ by at most 1 on at most 1e-4 of the elements (rounding-boundary ties only).
"""
import numpy as np
import pytest
import torch

from decode_attention_head_b200 import binding as bnd
from decode_attention_head_b200 import synth
from tests import harness as H

pytestmark = pytest.mark.gpu


def _tokens(rng, B, n, Hkv, outliers=True):
    x = rng.standard_normal((B, n, Hkv, 128))
    if outliers:
        x[..., [5, 40, 77, 119]] *= 20
    return x.astype(np.float16)


def _run(cfg, chunks, T, seed):
    rng = np.random.default_rng(seed)
    oc = H.oracle_cache_for(cfg)
    gc = bnd.KVCache(cfg)
    t_dev = H.to_dev(T)
    for n in chunks:
        k = _tokens(rng, cfg.batch, n, cfg.n_kv_heads)
        v = _tokens(rng, cfg.batch, n, cfg.n_kv_heads, outliers=False) * np.float16(2)
        oc.append(k, v, T)
        gc.append(H.to_dev(k), H.to_dev(v), t_dev)
    torch.cuda.synchronize()
    return oc, gc, H.download(gc)


CHUNKS = [1] * 40 + [37] + [1] * 19 + [300] + [1] * 7 + [2, 0, 1]


@pytest.mark.parametrize("bits,p_lo,p_hi,sink,keep,flush,chunk_max", [
    (2, 1.0, 99.0, 4, 32, 16, 1),
    (4, 0.5, 99.5, 4, 64, 16, 1),
    (2, 1.0, 99.0, 0, 0, 1, 1),
    (2, 0.5, 99.5, 2, 5, 7, 3),
    (4, 1.0, 99.0, 16, 8, 4, 2),
    (2, 2.0, 98.0, 4, 32, 16, 1),
])
def test_append_identity_transform_bit_exact(bits, p_lo, p_hi, sink, keep, flush, chunk_max):
    cfg = bnd.make_config(2, 2, 8, bits, 700, sink, keep, flush, chunk_max, p_lo, p_hi)
    T = np.broadcast_to(np.eye(128, dtype=np.float16), (2, 128, 128)).copy()
    oc, gc, g = _run(cfg, CHUNKS, T, seed=bits * 10 + sink)
    assert g["status"] == 0
    H.compare_caches(oc, g, cfg, gc.layout.ring_slots, exact=True)
    assert int(oc.S_quant[0]) > sink + 100


def test_append_random_transform_within_tolerance():
    wl = synth.WORKLOADS["tiny"]
    cfg = bnd.make_config(2, 2, 8, 2, 1200, 4, 32, 16, 1)
    T = np.stack([synth.key_transform(wl, 0, h).numpy() for h in range(2)])
    oc, gc, g = _run(cfg, [1] * 30 + [500] + [1] * 30 + [400] + [1] * 9, T, seed=3)
    st = H.compare_caches(oc, g, cfg, gc.layout.ring_slots, exact=False)
    assert st["code_maxdiff"] <= 1, st
    assert st["code_diff"] <= 1e-4 * st["code_elems"], st
    # k' near zero: fp32 (tensor-core) vs double accumulation can differ by a few fp16 ulps
    assert st["fp16_maxulp"] <= 8, st
    assert st["fp16_diff"] <= 2e-3 * st["fp16_elems"], st
    print(f"[append-random-T] {st}")
    assert st["param_diff"] <= 0.02 * st["param_tokens"], st


def test_append_values_untransformed_and_bulk_large():
    """A bulk chunk of several GEMM tiles with a ragged tail, identity-free T on keys only;
    values bypass the transform, so their codes must be bit-exact."""
    wl = synth.WORKLOADS["tiny"]
    cfg = bnd.make_config(1, 2, 2, 2, 3000, 4, 128, 16, 1)
    T = np.stack([synth.key_transform(wl, 0, h).numpy() for h in range(2)])
    oc, gc, g = _run(cfg, [2333, 1, 1, 600], T, seed=9)
    H.compare_caches(oc, g, cfg, gc.layout.ring_slots, exact=True, kinds=("v",))


def test_capacity_overflow_sets_status_and_skips():
    cfg = bnd.make_config(1, 1, 4, 2, 100, 4, 16, 16, 1)
    T = np.eye(128, dtype=np.float16)[None]
    oc, gc, g = _run(cfg, [90], T, seed=1)
    k = H.to_dev(np.ones((1, 20, 1, 128), np.float16))
    gc.append(k, k, H.to_dev(T))
    torch.cuda.synchronize()
    g2 = H.download(gc)
    assert g2["status"] & bnd.STATUS_OVERFLOW
    assert g2["S"][0, 0] == 90
    assert np.array_equal(g2["k_codes"], g["k_codes"])
    # a fitting append still works afterwards
    k = H.to_dev(np.ones((1, 10, 1, 128), np.float16))
    gc.append(k, k, H.to_dev(T))
    torch.cuda.synchronize()
    assert int(gc.lengths()[0][0, 0]) == 100
