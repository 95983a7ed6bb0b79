"""wushkv_step (append fused with the decode's preparation) against the same work done by
wushkv_append then wushkv_decode_attn, through the C ABI, on twin caches fed the same
tokens: the caches must stay bit-identical and the outputs agree to 1e-5; the outputs must
match the oracle's attention over the same (downloaded) cache, and the cache must match
the oracle's own within the general-transform bounds."""
import numpy as np
import pytest
import torch

from decode_attention_head_b200 import binding as bnd
from decode_attention_head_b200 import synth
from tests import harness as H

pytestmark = pytest.mark.gpu


def _tokens(rng, B, n, Hkv, scale=1.0):
    x = rng.standard_normal((B, n, Hkv, 128)) * scale
    x[..., [3, 50, 90]] *= 15
    return x.astype(np.float16)


def _assert_same_cache(ga, gb):
    da, db = H.download(ga), H.download(gb)
    for k in da:
        if k == "status":
            assert da[k] == db[k]
        else:
            a_, b_ = np.ascontiguousarray(da[k]), np.ascontiguousarray(db[k])
            assert a_.dtype == b_.dtype and np.array_equal(a_.view(np.uint8), b_.view(np.uint8)), k


@pytest.mark.parametrize("bits,Hkv,Hq,sink,keep,flush,chunk_max", [
    (2, 2, 8, 4, 32, 16, 1),
    (4, 2, 16, 4, 64, 16, 1),
    (2, 4, 4, 0, 8, 1, 1),
    (2, 1, 2, 2, 5, 7, 3),
])
def test_step_equals_append_then_decode(bits, Hkv, Hq, sink, keep, flush, chunk_max):
    B = 2
    cfg = bnd.make_config(B, Hkv, Hq, bits, 2000, sink, keep, flush, chunk_max)
    wl = synth.WORKLOADS["tiny"]
    T = np.stack([synth.key_transform(wl, 5, h).numpy() for h in range(Hkv)])
    t_dev = H.to_dev(T)
    tinv = bnd.compensation(torch.from_numpy(T)).cuda()
    scale = 1 / np.sqrt(128)
    ga, gb = bnd.KVCache(cfg), bnd.KVCache(cfg)
    oc = H.oracle_cache_for(cfg)
    rng = np.random.default_rng(bits * 7 + Hkv)
    # start from an empty cache: steps of 1 and chunk_max tokens, one bulk chunk, more steps
    plan = [1] * 5 + [chunk_max] * 3 + [700] + [1] * 40 + [chunk_max] * 2
    for i, n in enumerate(plan):
        k = _tokens(rng, B, n, Hkv)
        v = _tokens(rng, B, n, Hkv, 2.0)
        q = rng.standard_normal((B, Hq, 128)).astype(np.float16)
        kd, vd, qd = H.to_dev(k), H.to_dev(v), H.to_dev(q)
        out_a = ga.step(kd, vd, t_dev, qd, tinv, scale)
        gb.append(kd, vd, t_dev)
        out_b = gb.decode_attn(qd, tinv, scale)
        oc.append(k, v, T)
        torch.cuda.synchronize()
        err = (out_a - out_b).abs().max().item()
        assert err <= 1e-5, (i, n, err)
        if i % 10 == 0 or n > chunk_max:
            _assert_same_cache(ga, gb)
            # decode parity on the GPU's own cache (append differences are bounded below)
            H.assert_attention_close(out_a.cpu().numpy(), H.oracle_decode(H.oracle_cache_from_gpu(ga), q, T, scale))
    _assert_same_cache(ga, gb)
    assert ga.status() == 0
    st = H.compare_caches(oc, H.download(ga), cfg, ga.layout.ring_slots, exact=False)
    assert st["code_maxdiff"] <= 1 and st["code_diff"] <= 1e-4 * st["code_elems"], st
    assert st["fp16_maxulp"] <= 8 and st["param_diff"] <= 0.02 * st["param_tokens"], st


def test_step_refused_append_still_decodes():
    """At capacity the append is refused (STATUS_OVERFLOW) and the step's decode attends
    over the cache as it stands, like a plain decode."""
    cfg = bnd.make_config(1, 2, 8, 2, 300, 4, 32, 16, 1)
    T = np.broadcast_to(np.eye(128, dtype=np.float16), (2, 128, 128)).copy()
    t_dev = H.to_dev(T)
    tinv = bnd.compensation(torch.from_numpy(T)).cuda()
    rng = np.random.default_rng(3)
    g = bnd.KVCache(cfg)
    k = _tokens(rng, 1, 300, 2)
    g.append(H.to_dev(k), H.to_dev(k), t_dev)
    q = H.to_dev(rng.standard_normal((1, 8, 128)).astype(np.float16))
    ref = g.decode_attn(q, tinv, 0.1)
    one = H.to_dev(_tokens(rng, 1, 1, 2))
    out = g.step(one, one, t_dev, q, tinv, 0.1)
    torch.cuda.synchronize()
    assert g.status() & bnd.STATUS_OVERFLOW
    assert int(g.lengths()[0][0, 0]) == 300
    assert (out - ref).abs().max().item() <= 1e-5


def test_step_with_corrupt_state_is_isolated():
    """A fused step over a cache whose (sequence 1, KV head 0) state word is corrupt: that
    unit is reported (STATUS_BADSTATE), not appended to and decoded as empty; every other
    unit is appended to, advances its state and decodes like append + decode on a twin."""
    cfg = bnd.make_config(2, 2, 8, 2, 500, 4, 32, 16, 1)
    T = np.broadcast_to(np.eye(128, dtype=np.float16), (2, 128, 128)).copy()
    t_dev = H.to_dev(T)
    tinv = bnd.compensation(torch.from_numpy(T)).cuda()
    rng = np.random.default_rng(11)
    ga, gb = bnd.KVCache(cfg), bnd.KVCache(cfg)
    k = H.to_dev(_tokens(rng, 2, 300, 2))
    for g in (ga, gb):
        g.append(k, k, t_dev)
    units = 4
    for g in (ga, gb):
        g.state[: 2 * units].view(units, 2)[2, 0] = 10 ** 6
    for i in range(20):  # crosses a flush boundary of the healthy units
        one = H.to_dev(_tokens(rng, 2, 1, 2))
        q = H.to_dev(rng.standard_normal((2, 8, 128)).astype(np.float16))
        out_a = ga.step(one, one, t_dev, q, tinv, 0.1)
        gb.append(one, one, t_dev)
        out_b = gb.decode_attn(q, tinv, 0.1)
        torch.cuda.synchronize()
        assert torch.isfinite(out_a).all()
        assert torch.all(out_a[1, 0:4] == 0)
        assert (out_a - out_b).abs().max().item() <= 1e-5, i
    assert ga.status() & bnd.STATUS_BADSTATE
    sa = ga.state[: 2 * units].view(units, 2).cpu()
    sb = gb.state[: 2 * units].view(units, 2).cpu()
    assert torch.equal(sa, sb)
    assert int(sa[2, 0]) == 10 ** 6 and int(sa[0, 0]) == 320 and int(sa[3, 0]) == 320


def test_step_with_no_new_tokens_is_a_decode():
    """n_new = 0: the step appends nothing (a flush that is due still happens, as in
    wushkv_append) and its output equals wushkv_decode_attn over the same cache."""
    cfg = bnd.make_config(2, 2, 8, 2, 800, 4, 32, 16, 1)
    T = np.broadcast_to(np.eye(128, dtype=np.float16), (2, 128, 128)).copy()
    t_dev = H.to_dev(T)
    tinv = bnd.compensation(torch.from_numpy(T)).cuda()
    rng = np.random.default_rng(5)
    ga, gb = bnd.KVCache(cfg), bnd.KVCache(cfg)
    k = H.to_dev(_tokens(rng, 2, 300, 2))
    for g in (ga, gb):
        g.append(k, k, t_dev)
    empty = torch.empty(2, 0, 2, 128, dtype=torch.float16, device="cuda")
    q = H.to_dev(rng.standard_normal((2, 8, 128)).astype(np.float16))
    out_a = ga.step(empty, empty, t_dev, q, tinv, 0.1)
    gb.append(empty, empty, t_dev)
    out_b = gb.decode_attn(q, tinv, 0.1)
    torch.cuda.synchronize()
    assert ga.status() == 0 and gb.status() == 0
    assert (out_a - out_b).abs().max().item() <= 1e-5
    _assert_same_cache(ga, gb)
