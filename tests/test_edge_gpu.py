"""Edge cases of the GPU path through the C ABI: degenerate token rows (constant rows,
two-valued rows, signed zeros, fp16 subnormals, values near the fp16 limit) quantized
bit-exactly like the oracle, and corrupt state words reported (STATUS_BADSTATE) with the
affected (sequence, KV head) left untouched by the append and read as empty by the
decode, while the other units are served normally."""
import numpy as np
import pytest
import torch

from decode_attention_head_b200 import binding as bnd
from tests import harness as H

pytestmark = pytest.mark.gpu


def _degenerate_rows(rng, n, Hkv):
    """[1, n, Hkv, 128] fp16 rows cycling through the degenerate kinds."""
    x = np.zeros((1, n, Hkv, 128), np.float64)
    for t in range(n):
        for h in range(Hkv):
            kind = (t + h) % 7
            if kind == 0:
                x[0, t, h] = 1.5                                   # constant: s = 0
            elif kind == 1:
                x[0, t, h] = np.where(rng.random(128) < 0.5, -2.0, 3.0)  # two values
            elif kind == 2:
                x[0, t, h] = np.where(rng.random(128) < 0.5, -0.0, 0.0)  # signed zeros only
            elif kind == 3:
                x[0, t, h] = rng.integers(-50, 50, 128) * 2.0 ** -24    # fp16 subnormals
            elif kind == 4:
                x[0, t, h] = rng.uniform(-60000, 60000, 128)             # near the fp16 limit
            elif kind == 5:
                v = np.zeros(128)
                v[rng.integers(128)] = 7.0                               # one spike
                x[0, t, h] = v
            else:
                x[0, t, h] = rng.standard_normal(128)
    return x.astype(np.float16)


@pytest.mark.parametrize("bits,p_lo,p_hi", [(2, 1.0, 99.0), (4, 0.5, 99.5)])
def test_degenerate_rows_bit_exact(bits, p_lo, p_hi):
    cfg = bnd.make_config(1, 2, 8, bits, 1000, 4, 16, 8, 1, p_lo, p_hi)
    T = np.broadcast_to(np.eye(128, dtype=np.float16), (2, 128, 128)).copy()
    rng = np.random.default_rng(bits)
    oc = H.oracle_cache_for(cfg)
    gc = bnd.KVCache(cfg)
    t_dev = H.to_dev(T)
    for n in [1] * 30 + [200] + [1] * 20:
        k = _degenerate_rows(rng, n, 2)
        v = _degenerate_rows(rng, n, 2)
        oc.append(k, v, T)
        gc.append(H.to_dev(k), H.to_dev(v), t_dev)
    torch.cuda.synchronize()
    g = H.download(gc)
    assert g["status"] == 0
    H.compare_caches(oc, g, cfg, gc.layout.ring_slots, exact=True)
    q = rng.standard_normal((1, 8, 128)).astype(np.float16)
    tinv = bnd.compensation(torch.from_numpy(T)).cuda()
    out = gc.decode_attn(H.to_dev(q), tinv, 1 / np.sqrt(128))
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    # near-limit rows make logits large: compare relative to the output's scale
    ref = H.oracle_decode(H.oracle_cache_from_gpu(gc), q, T, 1 / np.sqrt(128))
    err = np.abs(out.cpu().numpy() - ref).max() / max(1.0, np.abs(ref).max())
    assert err <= 1e-3, err


def test_corrupt_state_is_reported_and_isolated():
    cfg = bnd.make_config(2, 2, 8, 2, 500, 4, 32, 16, 1)
    T = np.broadcast_to(np.eye(128, dtype=np.float16), (2, 128, 128)).copy()
    t_dev = H.to_dev(T)
    tinv = bnd.compensation(torch.from_numpy(T)).cuda()
    rng = np.random.default_rng(0)
    gc = bnd.KVCache(cfg)
    k = rng.standard_normal((2, 300, 2, 128)).astype(np.float16)
    gc.append(H.to_dev(k), H.to_dev(k), t_dev)
    torch.cuda.synchronize()
    q = H.to_dev(rng.standard_normal((2, 8, 128)).astype(np.float16))
    good = gc.decode_attn(q, tinv, 0.1).clone()
    # unit (sequence 1, KV head 0): S beyond the capacity
    units = 4
    st = gc.state[: 2 * units].view(units, 2)
    st[2, 0] = 10 ** 6
    one = H.to_dev(np.ones((2, 1, 2, 128), np.float16))
    gc.append(one, one, t_dev)
    out = gc.decode_attn(q, tinv, 0.1)
    torch.cuda.synchronize()
    assert gc.status() & bnd.STATUS_BADSTATE
    after = gc.state[: 2 * units].view(units, 2)
    assert int(after[2, 0]) == 10 ** 6            # the corrupt unit was not appended to
    assert int(after[0, 0]) == 301 and int(after[3, 0]) == 301
    assert torch.all(out[1, 0:4] == 0)           # its query heads read an empty cache
    assert torch.isfinite(out).all()
    # the other units attend over their (one token longer) caches as usual
    assert float((out[0] - good[0]).abs().max()) < 0.5
