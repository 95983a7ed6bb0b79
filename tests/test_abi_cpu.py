"""C-ABI checks that need no GPU: the library loads, exports every entry point the
header declares, sizes buffers as documented, and rejects bad arguments before any
device work."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wushkv.h")


@pytest.fixture(scope="module")
def bnd():
    from decode_attention_head_b200 import build
    build.build()
    from decode_attention_head_b200 import binding
    return binding


def test_exports_every_declared_symbol(bnd):
    text = open(HEADER).read()
    declared = set(re.findall(r"^\s*int\s+(wushkv_\w+)\s*\(", text, flags=re.M))
    assert declared == set(bnd.SYMBOLS)
    for name in declared:
        assert hasattr(bnd.lib, name)
    # the exported names of the .so, read from the dynamic symbol table via ctypes
    for name in declared:
        assert ctypes.cast(getattr(bnd.lib, name), ctypes.c_void_p).value


def test_layout_sizes(bnd):
    cfg = bnd.make_config(8, 8, 32, 2, 32768 + 1000, 4, 128, 16, 1)
    L = bnd.pack_layout(cfg)
    assert L.cap_alloc == 33792 and L.cap_alloc % 128 == 0
    assert L.code_bytes == 32
    assert L.ring_slots == 128 + 16 - 1 + 1
    assert L.codes_bytes == 64 * 33792 * 32
    assert L.params_bytes == 64 * 33792 * 4
    assert L.sink_bytes == 64 * 4 * 128 * 2
    assert L.ring_bytes == 64 * 144 * 128 * 2
    assert L.state_bytes >= (2 * 64 + 1) * 4
    assert L.split_tokens % 128 == 0 and L.n_splits * L.split_tokens >= L.cap_alloc
    assert L.workspace_bytes > 0
    # keys canonical, values in the 16-position group layout the header documents
    assert L.code_order == bnd.CODE_ORDER_VGROUP16 == 1
    cfg4 = bnd.make_config(64, 32, 32, 4, 8192, 4, 64, 16, 1, 0.5, 99.5)
    L4 = bnd.pack_layout(cfg4)
    assert L4.code_bytes == 64 and L4.codes_bytes == 64 * 32 * 8192 * 64


@pytest.mark.parametrize("field,value,code", [
    ("head_dim", 64, -2), ("bits", 3, -2), ("n_q_heads", 24, -2), ("n_q_heads", 7, -1), ("n_q_heads", 12, -2),
    ("s_flush", 0, -1), ("chunk_max", 0, -1), ("capacity", 0, -1), ("s_sink", -1, -1),
    ("p_lo", 99.0, -1), ("p_hi", 101.0, -1), ("p_lo", 10.0, -2)])
def test_bad_configs_rejected(bnd, field, value, code):
    cfg = bnd.make_config(2, 2, 8, 2, 1000, 4, 32, 16, 1)
    setattr(cfg, field, value)
    out = bnd.Layout()
    assert bnd.lib.wushkv_pack_layout(ctypes.byref(cfg), ctypes.byref(out)) == code


def test_bad_pointers_rejected_before_device_work(bnd):
    cfg = bnd.make_config(1, 1, 4, 2, 256, 4, 32, 16, 1)
    bufs = bnd.CacheBufs()          # all null
    rc = bnd.lib.wushkv_append(ctypes.byref(cfg), ctypes.byref(bufs), None, None, 1, None, None)
    assert rc == bnd.EINVAL
    rc = bnd.lib.wushkv_decode_attn(ctypes.byref(cfg), ctypes.byref(bufs), None, None, ctypes.c_float(0.1), 0,
                                    None, None, None)
    assert rc == bnd.EINVAL
    rc = bnd.lib.wushkv_step(ctypes.byref(cfg), ctypes.byref(bufs), None, None, 1, None, None, None,
                             ctypes.c_float(0.1), 0, None, None, None)
    assert rc == bnd.EINVAL
    rc = bnd.lib.wushkv_decode_attn_static(ctypes.byref(cfg), ctypes.byref(bufs), None, None, ctypes.c_float(0.1),
                                           0, None, None)
    assert rc == bnd.EINVAL
    assert bnd.lib.wushkv_pack_layout(None, None) == bnd.EINVAL


def test_static_scratch_limit_checked_on_the_host(bnd):
    """A configuration needing more scratch than the library's array is refused before any
    CUDA call (the pointers are never dereferenced: the check comes first)."""
    cfg = bnd.make_config(512, 8, 64, 2, 128, 4, 32, 16, 1)
    assert bnd.pack_layout(cfg).workspace_bytes > bnd.STATIC_SCRATCH_BYTES
    fake = 1 << 20  # aligned, never touched
    bufs = bnd.CacheBufs(*([fake] * 9))
    rc = bnd.lib.wushkv_decode_attn_static(ctypes.byref(cfg), ctypes.byref(bufs), fake, fake, ctypes.c_float(0.1),
                                           0, fake, None)
    assert rc == bnd.ESCRATCH


def test_compensation_inverts_fp16_transform(bnd):
    rng = np.random.default_rng(7)
    q, r = np.linalg.qr(rng.standard_normal((3, 128, 128)))
    t = (q * rng.uniform(0.5, 2, (3, 1, 128))).astype(np.float16)
    inv = bnd.compensation(torch.from_numpy(t)).numpy()
    ref = np.linalg.inv(t.astype(np.float64))
    np.testing.assert_allclose(inv, ref, rtol=0, atol=1e-5 * np.abs(ref).max())
    eye = np.einsum("hij,hjk->hik", t.astype(np.float64), inv.astype(np.float64))
    np.testing.assert_allclose(eye, np.broadcast_to(np.eye(128), eye.shape), atol=1e-4)


def test_compensation_rejects_singular(bnd):
    t = torch.zeros(1, 128, 128, dtype=torch.float16)
    with pytest.raises(bnd.WushKVError):
        bnd.compensation(t)


def test_hadamard_helper_and_transform_field(bnd):
    """wushkv_hadamard fills H (orthonormal, symmetric, +-1/sqrt(128) by popcount parity);
    an unknown transform kind is rejected."""
    import scipy.linalg
    h = bnd.hadamard_compensation(2).numpy()
    ref = (scipy.linalg.hadamard(128) / np.sqrt(128)).astype(np.float32)
    np.testing.assert_array_equal(h[0], ref)
    np.testing.assert_array_equal(h[1], ref)
    cfg = bnd.make_config(2, 2, 8, 2, 1000, 4, 32, 16, 1, transform=bnd.TRANSFORM_HADAMARD)
    assert bnd.pack_layout(cfg).cap_alloc == 1024
    cfg.transform = 2
    assert bnd.lib.wushkv_pack_layout(ctypes.byref(cfg), ctypes.byref(bnd.Layout())) == bnd.EINVAL


def test_rms_quantizer_config_checks(bnd):
    ok = bnd.make_config(1, 1, 4, 2, 256, 4, 32, 16, 1, quantizer=bnd.QUANT_RMS, clip_alpha=1.4936)
    assert bnd.lib.wushkv_pack_layout(ctypes.byref(ok), ctypes.byref(bnd.Layout())) == bnd.OK
    # percentiles are not used by the RMS quantizer, so ranks outside the supported four are fine
    ok.p_lo, ok.p_hi = 10.0, 90.0
    assert bnd.lib.wushkv_pack_layout(ctypes.byref(ok), ctypes.byref(bnd.Layout())) == bnd.OK
    for alpha in (0.0, -1.0, float("inf")):
        bad = bnd.make_config(1, 1, 4, 2, 256, 4, 32, 16, 1, quantizer=bnd.QUANT_RMS, clip_alpha=alpha)
        assert bnd.lib.wushkv_pack_layout(ctypes.byref(bad), ctypes.byref(bnd.Layout())) == bnd.EINVAL
    bad = bnd.make_config(1, 1, 4, 2, 256, 4, 32, 16, 1)
    bad.quantizer = 7
    assert bnd.lib.wushkv_pack_layout(ctypes.byref(bad), ctypes.byref(bnd.Layout())) == bnd.EINVAL


def test_gram_accumulate_argument_checks(bnd):
    """wushkv_gram_accumulate validates on the host before any CUDA call; zero tokens
    queue nothing (the aligned fake pointers are never dereferenced)."""
    f = bnd.lib.wushkv_gram_accumulate
    fake = 1 << 20
    assert f(None, 10, 2, fake, None) == bnd.EINVAL
    assert f(fake, 10, 2, None, None) == bnd.EINVAL
    assert f(fake + 8, 10, 2, fake, None) == bnd.EINVAL
    assert f(fake, 10, 2, fake + 8, None) == bnd.EINVAL
    assert f(fake, -1, 2, fake, None) == bnd.EINVAL
    assert f(fake, 10, 0, fake, None) == bnd.EINVAL
    assert f(fake, 10, 65536, fake, None) == bnd.EINVAL
    assert f(fake, (1 << 40) // 8 + 1, 8, fake, None) == bnd.EINVAL
    assert f(fake, 0, 8, fake, None) == bnd.OK
    assert f(None, 0, 8, fake, None) == bnd.OK
    assert f(None, 0, 8, None, None) == bnd.EINVAL
    with pytest.raises(bnd.WushKVError):
        bnd.gram_accumulate(torch.zeros(4, 2, 128, dtype=torch.float32), torch.zeros(2, 128, 128, dtype=torch.float64))
    with pytest.raises(bnd.WushKVError):
        bnd.gram_accumulate(torch.zeros(4, 2, 128, dtype=torch.float16), torch.zeros(3, 128, 128, dtype=torch.float64))
    # well-formed but on the host: refused before the library is called
    with pytest.raises(bnd.WushKVError, match="CUDA"):
        bnd.gram_accumulate(torch.zeros(4, 2, 128, dtype=torch.float16), torch.zeros(2, 128, 128, dtype=torch.float64))


def test_binding_refuses_host_tensors(bnd):
    """The check every binding entry runs before handing tensors to the library: host
    tensors are refused (a host pointer on the device would fault), None is allowed."""
    bnd._require_cuda(None)
    with pytest.raises(bnd.WushKVError, match="CUDA"):
        bnd._require_cuda(None, torch.zeros(1))


def test_decode_split_policy(bnd):
    """The decode's work split: n_split items per (sequence, KV head) filling the B200's
    CTA slots (148 SMs, 4 CTAs each, 3 for 8 query heads per KV head), in clusters of two
    consecutive items when n_split is even, never more than 128 items."""
    from decode_attention_head_b200 import synth
    expect = {"llama3-8b-layer": (9, 1), "qwen3-8b-layer": (74, 2), "mha-32l": (2, 2),
              "prefill-append-decode": (13, 1), "tiny": (128, 2)}
    for name, wl in synth.WORKLOADS.items():
        L = bnd.pack_layout(bnd.config_for_workload(wl, extra_capacity=64))
        assert (L.n_splits, L.decode_cluster) == expect[name], name
        # the grid interleaves the units where a unit's items fill a quarter of a round of
        # CTAs (148 SMs): here the Qwen3-8B layer's one sequence and the tiny parity case
        assert L.decode_interleave == (1 if L.n_splits * 4 >= 148 else 0), name
        assert L.decode_interleave == (name in ("qwen3-8b-layer", "tiny")), name
    for B, Hkv, Hq in [(1, 1, 1), (1, 8, 64), (3, 8, 32), (16, 8, 32), (64, 32, 32), (256, 8, 8)]:
        L = bnd.pack_layout(bnd.make_config(B, Hkv, Hq, 2, 4096, 4, 32, 16, 1))
        slots = 148 * (3 if Hq // Hkv == 8 else 4)
        assert 1 <= L.n_splits <= 128 and L.decode_cluster == (2 if L.n_splits % 2 == 0 else 1)
        if B * Hkv * L.n_splits > slots:  # more than one wave only when one item per unit overfills it
            assert L.n_splits <= 4


def test_workspace_counters_cover_every_chunk_launch(bnd):
    """Every layout of a configuration reserves the same leading completion counters: one per
    virtual unit of its largest chunk-attention launch (up to 32 blocks of chunk tokens per
    (sequence, KV head), no more than chunk_max, and no more grid rows than 65535), so that
    decode, step and chunk calls can share one workspace.  The decode layout grows by exactly
    that reservation as chunk_max grows; the rest of it does not depend on chunk_max."""
    def up(x):
        return (x + 255) // 256 * 256
    for B, Hkv, Hq in [(8, 8, 32), (2, 2, 8), (1, 1, 8), (600, 64, 64)]:
        U = B * Hkv
        base = bnd.pack_layout(bnd.make_config(B, Hkv, Hq, 2, 4096, 4, 32, 16, 1))
        for cmax in (2, 8, 40):
            L = bnd.pack_layout(bnd.make_config(B, Hkv, Hq, 2, 4096, 4, 32, 16, cmax))
            mp = max(1, min(32, cmax, 65535 // U))
            assert L.workspace_bytes - base.workspace_bytes == up(4 * U * mp) - up(4 * U), (B, Hkv, cmax)
            assert L.chunk_workspace_bytes >= L.workspace_bytes
