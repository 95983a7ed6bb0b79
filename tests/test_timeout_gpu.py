"""The bounded in-kernel waits, made to run out on purpose without faulting anything.

wushkv_decode_attn_test_timeout shortens the decode kernel's wait limit and withholds the
issue of one pipeline stage (the copy is never started, so no copy is in flight when a
warp gives up).  The call must return, the status word must carry STATUS_TIMEOUT, no
output row may be written (an aborted work item's cluster writes no output), the
workspace's completion counters must be back at zero, and the next ordinary call on the
same cache and workspace must be exact again.
"""
import numpy as np
import pytest
import torch

from decode_attention_head_b200 import binding as bnd
from decode_attention_head_b200 import synth
from tests import harness as H

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bits,g", [(2, 4), (4, 1), (2, 8)])
def test_withheld_stage_times_out_cleanly(bits, g):
    B, Hkv = 2, 2
    cfg = bnd.make_config(B, Hkv, Hkv * g, bits, 3000, 4, 32, 16, 1)
    wl = synth.WORKLOADS["tiny"]
    T = np.stack([synth.key_transform(wl, 1, h).numpy() for h in range(Hkv)])
    rng = np.random.default_rng(bits * 10 + g)
    gc = bnd.KVCache(cfg)
    kv = [H.to_dev(rng.standard_normal((B, 2600, Hkv, 128)).astype(np.float16)) for _ in range(2)]
    gc.append(kv[0], kv[1], H.to_dev(T))
    q = H.to_dev(rng.standard_normal((B, Hkv * g, 128)).astype(np.float16))
    tinv = bnd.compensation(torch.from_numpy(T)).cuda()
    scale = 1 / np.sqrt(128)
    ref = gc.decode_attn(q, tinv, scale)
    torch.cuda.synchronize()
    assert gc.status() == 0

    out = torch.full_like(ref, float("nan"))
    gc.decode_attn_test_timeout(q, tinv, scale, out, withhold_stage=0, wait_limit_cycles=2_000_000)
    torch.cuda.synchronize()
    assert gc.status() & bnd.STATUS_TIMEOUT
    assert torch.isnan(out).all(), "an aborted call must not write plausible-looking output"
    # the workspace's completion counters (its first 4 * units bytes) are back at zero: the
    # next call needs no clearing
    assert not gc.workspace[:4 * gc.units].any()

    gc.state[2 * gc.units] = 0  # clear the status word (after the (S, S_quant) pairs)
    again = gc.decode_attn(q, tinv, scale)
    torch.cuda.synchronize()
    assert gc.status() == 0
    assert torch.equal(again, ref)
    assert not gc.workspace[:4 * gc.units].any()


def test_hook_arguments_are_checked():
    cfg = bnd.make_config(1, 1, 4, 2, 256, 4, 32, 16, 1)
    gc = bnd.KVCache(cfg)
    q = torch.zeros(1, 4, 128, dtype=torch.float16, device="cuda")
    out = torch.zeros(1, 4, 128, device="cuda")
    tinv = torch.eye(128, device="cuda")[None].contiguous()
    for stage, limit in [(-2, 10_000), (0, 10), (0, 1 << 40)]:
        with pytest.raises(bnd.WushKVError):
            gc.decode_attn_test_timeout(q, tinv, 0.1, out, stage, limit)
