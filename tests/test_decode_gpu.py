"""GPU decode attention vs the oracle, through the C ABI, on identical caches: the oracle
builds the cache from seeded inputs, the test writes it into the library's buffers
(documented layout), and both sides attend over it.  Tolerance: 2e-3 max abs and 1e-3
relative (2-norm per output row)."""
import numpy as np
import pytest
import torch

from decode_attention_head_b200 import binding as bnd
from decode_attention_head_b200 import synth
from tests import harness as H

pytestmark = pytest.mark.gpu


def _build(cfg, S, seed, T, chunk=256, v_t=True):
    rng = np.random.default_rng(seed)
    oc = H.oracle_cache_for(cfg)
    done = 0
    while done < S:
        n = min(chunk, S - done)
        if S - done <= 2:
            n = 1                              # finish with small appends (deferred flush state)
        k = rng.standard_normal((cfg.batch, n, cfg.n_kv_heads, 128))
        k[..., [3, 17, 64, 100]] *= 20
        if v_t:
            z = rng.standard_normal((cfg.batch, n, cfg.n_kv_heads, 128))
            chi = (rng.standard_normal((5, cfg.batch, n, cfg.n_kv_heads, 128)) ** 2).sum(0)
            v = z / np.sqrt(chi / 5)
        else:
            v = rng.standard_normal((cfg.batch, n, cfg.n_kv_heads, 128))
        oc.append(k.astype(np.float16), v.astype(np.float16), T)
        done += n
    return oc


def _transform(Hkv, seed, identity=False):
    if identity:
        return np.broadcast_to(np.eye(128, dtype=np.float16), (Hkv, 128, 128)).copy()
    rng = np.random.default_rng(seed + 1000)
    out = []
    for _ in range(Hkv):
        q, r = np.linalg.qr(rng.standard_normal((128, 128)))
        out.append((q * np.sign(np.diag(r))) * rng.uniform(0.5, 2, 128))
    return np.stack(out).astype(np.float16)


def _decode_case(cfg, S, seed, identity=False, out_fp16=False, capacity_variants=()):
    T = _transform(cfg.n_kv_heads, seed, identity)
    oc = _build(cfg, S, seed, T)
    rng = np.random.default_rng(seed + 7)
    q = rng.standard_normal((cfg.batch, cfg.n_q_heads, 128)).astype(np.float16)
    scale = 1 / np.sqrt(128)
    ref = H.oracle_decode(oc, q, T, scale)
    tinv = bnd.compensation(torch.from_numpy(T)).cuda()
    outs = []
    for cap in (cfg.capacity,) + tuple(capacity_variants):
        c2 = bnd.make_config(cfg.batch, cfg.n_kv_heads, cfg.n_q_heads, cfg.bits, cap, cfg.s_sink, cfg.s_keep,
                             cfg.s_flush, cfg.chunk_max, cfg.p_lo, cfg.p_hi)
        gc = bnd.KVCache(c2)
        H.upload(oc, gc)
        out = gc.decode_attn(H.to_dev(q), tinv, scale, out_fp16=out_fp16)
        torch.cuda.synchronize()
        outs.append(out.float().cpu().numpy())
        status = gc.status()
    return ref, outs, status, oc


@pytest.mark.parametrize("bits,G,sink,keep,flush,S,p", [
    (2, 4, 4, 32, 16, 512, (1.0, 99.0)),      # the tiny workload's shape
    (2, 4, 4, 128, 16, 4567, (1.0, 99.0)),    # several tiles and items, ragged tail
    (2, 1, 4, 32, 16, 1000, (1.0, 99.0)),
    (2, 2, 4, 32, 16, 1000, (1.0, 99.0)),
    (2, 8, 4, 128, 16, 3000, (1.0, 99.0)),
    (4, 4, 4, 64, 16, 2100, (0.5, 99.5)),
    (4, 1, 4, 64, 16, 1500, (0.5, 99.5)),
    (4, 8, 4, 64, 16, 900, (0.5, 99.5)),
    (2, 4, 0, 0, 1, 700, (1.0, 99.0)),        # no windows at all
    (2, 4, 16, 8, 7, 333, (0.5, 99.5)),
])
def test_decode_matches_oracle(bits, G, sink, keep, flush, S, p):
    cfg = bnd.make_config(2, 2, 2 * G, bits, S + 64, sink, keep, flush, 1, *p)
    ref, outs, status, oc = _decode_case(cfg, S, seed=bits * 100 + G * 10 + sink)
    assert status == 0
    assert int(oc.S_quant.max()) > 0 or keep + sink >= S
    H.assert_attention_close(outs[0], ref)


@pytest.mark.parametrize("S", [1, 3, 4, 36, 60])
def test_decode_windows_only_and_tiny_lengths(S):
    cfg = bnd.make_config(1, 2, 8, 2, 256, 4, 32, 16, 1)
    ref, outs, status, oc = _decode_case(cfg, S, seed=S)
    H.assert_attention_close(outs[0], ref)


def test_decode_empty_sequence_gives_zeros_and_status():
    cfg = bnd.make_config(1, 1, 4, 2, 256, 4, 32, 16, 1)
    gc = bnd.KVCache(cfg)
    tinv = torch.eye(128).unsqueeze(0).cuda()
    q = torch.ones(1, 4, 128, dtype=torch.float16, device="cuda")
    out = gc.decode_attn(q, tinv, 0.1)
    torch.cuda.synchronize()
    assert not out.any()
    assert gc.status() & bnd.STATUS_EMPTY


def test_decode_identity_transform_and_fp16_output():
    cfg = bnd.make_config(2, 2, 8, 2, 3000, 4, 128, 16, 1)
    ref, outs, _, _ = _decode_case(cfg, 2500, seed=5, identity=True, out_fp16=True)
    H.assert_attention_close(outs[0], ref, atol=2e-3, rtol=2e-3)   # fp16 output rounding


def test_decode_invariant_to_work_split():
    """Different capacities give different split policies; same cache, same answer."""
    cfg = bnd.make_config(1, 2, 8, 2, 9000, 4, 128, 16, 1)
    ref, outs, _, _ = _decode_case(cfg, 8000, seed=11, capacity_variants=(8064, 40000, 150000))
    for o in outs:
        H.assert_attention_close(o, ref)
    for o in outs[1:]:
        assert np.abs(o - outs[0]).max() < 1e-4


def test_decode_tiny_workload_synth_inputs():
    """The tiny workload exactly as specified (512 tokens, GQA 4, sink 4 + keep 32, seed 0)."""
    wl = synth.WORKLOADS["tiny"]
    cfg = bnd.config_for_workload(wl, extra_capacity=64)
    T = synth.key_transforms(wl).numpy()
    oc = H.oracle_cache_for(cfg)
    k = synth.batch_tokens(wl, 0, 0, wl.context, which="k").numpy()
    v = synth.batch_tokens(wl, 0, 0, wl.context, which="v").numpy()
    for t0 in range(0, wl.context, 16):
        oc.append(k[:, t0:t0 + 16], v[:, t0:t0 + 16], T)
    q = synth.batch_queries(wl, 0, wl.context - 1).numpy()
    ref = H.oracle_decode(oc, q, T, synth.default_softmax_scale())
    gc = bnd.KVCache(cfg)
    H.upload(oc, gc)
    out = gc.decode_attn(H.to_dev(q), bnd.compensation(torch.from_numpy(T)).cuda(), synth.default_softmax_scale())
    torch.cuda.synchronize()
    H.assert_attention_close(out.cpu().numpy(), ref)
