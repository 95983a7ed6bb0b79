"""wushkv_decode_attn_static (library-owned scratch, no allocation) against
wushkv_decode_attn (caller workspace), through the C ABI.

Collected last on purpose: it must pass both alone in a fresh process and after every
other test has used the device.  Three calls in a row on two configurations of
different size check that what one call leaves in the shared scratch array does not
leak into the next, and the free device memory must not move across the calls.
"""
import numpy as np
import pytest
import torch

from decode_attention_head_b200 import build

build.build()

from decode_attention_head_b200 import binding as bnd  # noqa: E402
from decode_attention_head_b200 import synth  # noqa: E402
from oracle import attention as oatt  # noqa: E402
from tests import harness as H  # noqa: E402
from tests.harness import ATOL  # noqa: E402

pytestmark = pytest.mark.gpu


def _filled_cache(cfg, n_bulk, n_single, seed):
    """A cache filled by one bulk append and `n_single` one-token appends of seeded data."""
    rng = np.random.default_rng(seed)
    wl = synth.WORKLOADS["tiny"]
    t_k = torch.stack([synth.key_transform(wl, seed, h) for h in range(cfg.n_kv_heads)])
    gc = bnd.KVCache(cfg)
    gc.t_k_host = t_k.numpy()
    t_dev = t_k.cuda()

    def tok(n, scale):
        x = rng.standard_normal((cfg.batch, n, cfg.n_kv_heads, 128)) * scale
        return torch.from_numpy(x.astype(np.float16)).cuda()

    gc.append(tok(n_bulk, 1.0), tok(n_bulk, 2.0), t_dev)
    for _ in range(n_single):
        gc.append(tok(1, 1.0), tok(1, 2.0), t_dev)
    q = tok(cfg.n_q_heads // cfg.n_kv_heads, 1.0).view(cfg.batch, cfg.n_q_heads, 128)
    t_inv = bnd.compensation(t_k).cuda()
    torch.cuda.synchronize()
    assert gc.status() == 0
    return gc, q, t_inv


SCALE = 1.0 / np.sqrt(128.0)


def _static(case, out_dtype):
    gc, q, t_inv = case
    out = torch.full(q.shape, float("nan"), dtype=out_dtype, device=q.device)
    return out, lambda: gc.decode_attn_static(q, t_inv, SCALE, out)


def _compare(case, out, ref):
    """The same kernels run on the same inputs with the scratch in another place: the result
    must be the workspace path's bit for bit (a stale-scratch leak of any size fails), and
    the oracle's within the attention tolerance."""
    gc, q = case[0], case[1]
    assert gc.status() == 0
    err = (out.float() - ref.float()).abs().max().item()
    print(f"[no-alloc] units={gc.units} splits={gc.layout.n_splits} dtype={out.dtype} max|diff|={err:.3g}")
    assert np.isfinite(err) and err <= ATOL
    assert torch.equal(out, ref)
    if out.dtype == torch.float32:
        want = oatt.decode(H.oracle_cache_from_gpu(gc), q.cpu().numpy(), gc.t_k_host, SCALE)
        H.assert_attention_close(out.cpu().numpy(), want)


def test_static_scratch_matches_workspace_path():
    small = bnd.make_config(2, 2, 8, 2, 3000, 4, 32, 16, 1)
    large = bnd.make_config(4, 4, 16, 4, 5000, 4, 64, 16, 1, 0.5, 99.5)
    assert bnd.pack_layout(large).workspace_bytes > bnd.pack_layout(small).workspace_bytes
    assert bnd.pack_layout(large).workspace_bytes <= bnd.STATIC_SCRATCH_BYTES
    a = _filled_cache(small, 2500, 40, seed=1)
    b = _filled_cache(large, 4400, 25, seed=2)
    ref_a = a[0].decode_attn(a[1], a[2], SCALE)
    ref_b = b[0].decode_attn(b[1], b[2], SCALE, out_fp16=True)

    # first call on this device: looks up the scratch array's address (and loads it)
    out0, call0 = _static(a, torch.float32)
    call0()
    torch.cuda.synchronize()
    _compare(a, out0, ref_a)

    # then calls in a row on different configurations: nothing allocated, results unchanged
    out1, call1 = _static(b, torch.float16)
    out2, call2 = _static(a, torch.float32)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    call1()
    call2()
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    _compare(b, out1, ref_b)
    _compare(a, out2, ref_a)


def test_static_scratch_rejects_oversized_configuration():
    cfg = bnd.make_config(512, 8, 64, 2, 128, 4, 32, 16, 1)
    assert bnd.pack_layout(cfg).workspace_bytes > bnd.STATIC_SCRATCH_BYTES
    gc = bnd.KVCache(cfg)
    q = torch.zeros(cfg.batch, cfg.n_q_heads, 128, dtype=torch.float16, device="cuda")
    t_inv = torch.eye(128, device="cuda").expand(cfg.n_kv_heads, 128, 128).contiguous()
    out = torch.zeros(q.shape, dtype=torch.float32, device="cuda")
    with pytest.raises(bnd.WushKVError, match="static scratch"):
        gc.decode_attn_static(q, t_inv, 0.1, out)
    torch.cuda.synchronize()
    assert bool((out == 0).all())
