"""wushkv_step_prep (raw q / k; per-head RMSNorm and RoPE inside the step's kernels)
against the oracle (oracle/rope.py then the cache and attention oracles), through the
C ABI.  Identity T_K keeps the post-RoPE keys visible in the fp16 windows, so they are
compared directly with the oracle's: the GPU rotates in fp32 (angles reduced in fp64) and
the oracle in float64, so a value next to an fp16 rounding tie may differ by one ulp of
the rotated pair's magnitude.
Decode parity is measured on the GPU's own cache with the oracle's rotated query."""
import numpy as np
import pytest
import torch

from decode_attention_head_b200 import binding as bnd
from oracle import rope as orope
from tests import harness as H

pytestmark = pytest.mark.gpu


def _ulps(a, b):
    ai = np.asarray(a, np.float16).view(np.int16).astype(np.int32)
    bi = np.asarray(b, np.float16).view(np.int16).astype(np.int32)
    return np.abs(ai - bi)


@pytest.mark.parametrize("bits,Hkv,Hq,theta,norm", [
    (2, 2, 8, 1e6, True),
    (4, 1, 8, 1e4, False),
    (2, 2, 4, 5e5, True),
])
def test_step_prep_matches_oracle(bits, Hkv, Hq, theta, norm):
    B = 2
    cfg = bnd.make_config(B, Hkv, Hq, bits, 3000, 4, 32, 16, 1)
    rng = np.random.default_rng(bits * 11 + Hq)
    T = np.broadcast_to(np.eye(128, dtype=np.float16), (Hkv, 128, 128)).copy()
    t_dev = H.to_dev(T)
    tinv = bnd.compensation(torch.from_numpy(T)).cuda()
    qg = rng.uniform(0.5, 1.5, 128).astype(np.float16) if norm else None
    kg = rng.uniform(0.5, 1.5, 128).astype(np.float16) if norm else None
    qg_d = H.to_dev(qg) if norm else None
    kg_d = H.to_dev(kg) if norm else None
    eps = 1e-6
    scale = 1 / np.sqrt(128)
    gc = bnd.KVCache(cfg)
    oc = H.oracle_cache_for(cfg)
    S = 0
    ulp_max, ulp_cnt, n_cmp = 0, 0, 0
    for i, n in enumerate([1] * 30 + [300] + [1] * 25 + [700] + [1] * 5):
        k_raw = (rng.standard_normal((B, n, Hkv, 128)) * 3).astype(np.float16)
        v = rng.standard_normal((B, n, Hkv, 128)).astype(np.float16)
        q_raw = (rng.standard_normal((B, Hq, 128)) * 3).astype(np.float16)
        out = gc.step_prep(H.to_dev(k_raw), H.to_dev(v), t_dev, H.to_dev(q_raw), tinv, scale, theta, qg_d, kg_d, eps)
        pos = (S + np.arange(n))[None, :, None]
        k_rope = orope.prepare(k_raw, pos, theta, kg, eps, norm)
        q_rope = orope.prepare(q_raw, S + n - 1, theta, qg, eps, norm)
        oc.append(k_rope, v, T)
        S += n
        torch.cuda.synchronize()
        assert gc.status() == 0
        g = H.download(gc)
        # post-RoPE keys in the windows: sink and recent ring (identity T_K: k' = k)
        for b in range(B):
            Sq = int(g["Sq"][b, 0])
            ns = min(cfg.s_sink, S)
            rpos = np.arange(max(Sq, cfg.s_sink), S)
            gk = np.concatenate([g["k_sink"][b][:, :ns], g["k_ring"][b][:, rpos % gc.layout.ring_slots]], axis=1)
            ok = np.concatenate([oc.k_store[b][:, :ns], oc.k_store[b][:, rpos]], axis=1)
            u = _ulps(gk, ok)
            ulp_cnt += int((u != 0).sum())
            n_cmp += u.size
            # a rotated value is a difference of two products; where they nearly cancel the
            # result is small and its own ulp is finer than the rounding error of the
            # operands, so the error is measured in ulps of the rotated pair's magnitude
            okf = ok.astype(np.float64)
            pair = np.hypot(okf, np.roll(okf, 64, axis=-1))
            ulp_pair = np.exp2(np.floor(np.log2(np.maximum(pair, 2.0 ** -14))) - 10)
            err = np.abs(gk.astype(np.float64) - okf) / ulp_pair
            ulp_max = max(ulp_max, float(err.max()))
        if i % 8 == 0 or n > 1:
            ref = H.oracle_decode(H.oracle_cache_from_gpu(gc), q_rope, T, scale)
            H.assert_attention_close(out.cpu().numpy(), ref)
    print(f"[prep] post-RoPE keys: max error {ulp_max:.2f} ulps of the pair magnitude, "
          f"{ulp_cnt} of {n_cmp} values differ")
    assert ulp_max <= 1.0 and ulp_cnt <= 2e-3 * n_cmp
    st = H.compare_caches(oc, H.download(gc), cfg, gc.layout.ring_slots, exact=False)
    print(f"[prep] cache vs oracle: {st}")
    assert st["code_maxdiff"] <= 1 and st["code_diff"] <= 1e-4 * st["code_elems"], st
    assert st["param_diff"] <= 0.02 * st["param_tokens"], st
    # the values pass through untouched
    assert np.array_equal(H.download(gc)["v_sink"].view(np.uint16), oc.v_store[:, :, :cfg.s_sink].view(np.uint16))


def test_step_prep_rejects_bad_spec():
    cfg = bnd.make_config(1, 1, 4, 2, 256, 4, 32, 16, 1)
    gc = bnd.KVCache(cfg)
    z = torch.zeros(1, 1, 1, 128, dtype=torch.float16, device="cuda")
    q = torch.zeros(1, 4, 128, dtype=torch.float16, device="cuda")
    T = torch.eye(128, dtype=torch.float16, device="cuda")[None]
    tinv = torch.eye(128, device="cuda")[None].contiguous()
    with pytest.raises(bnd.WushKVError):
        gc.step_prep(z, z, T, q, tinv, 0.1, rope_theta=1.0)
    g = torch.ones(128, dtype=torch.float16, device="cuda")
    with pytest.raises(bnd.WushKVError):
        gc.step_prep(z, z, T, q, tinv, 0.1, rope_theta=1e4, k_norm_gain=g, norm_eps=0.0)
    torch.cuda.synchronize()
    assert int(gc.lengths()[0][0, 0]) == 0
