"""Chunked prefill attention (wushkv_chunk_attn) against the oracle, through the C ABI:
after each append of a chunk of n <= chunk_max tokens (still in the fp16 window), the
chunk's n queries attend causally -- query t of the chunk sees positions up to its own --
and must match exact softmax attention over the same (downloaded) cache truncated at that
position.  A one-token chunk must equal wushkv_decode_attn."""
import numpy as np
import pytest
import torch

from decode_attention_head_b200 import binding as bnd
from decode_attention_head_b200 import synth
from oracle import attention as oatt
from tests import harness as H

pytestmark = pytest.mark.gpu


def ticket_words(cfg, B, Hkv):
    """The completion counters at the start of every workspace layout: one per virtual unit
    of the largest chunk-attention launch (blocks of chunk tokens run as up to 32 grid rows
    per (sequence, KV head))."""
    units = B * Hkv
    return units * max(1, min(32, cfg.chunk_max, 65535 // units))


# chunk lengths cover one block per launch, several equal blocks in one launch (8 tokens at
# g = 4: four blocks of two; 16 at g = 1: two blocks of eight; 4 at g = 8: four blocks of
# one), ragged remainders taking further launches (7 at g = 4: three blocks of two, then
# one token), and more blocks than one launch takes (40 at g = 8: 32 blocks, then 8)
@pytest.mark.parametrize("bits,Hkv,Hq,chunk", [(2, 2, 8, 8), (2, 2, 2, 16), (4, 1, 8, 4), (2, 2, 4, 3),
                                               (2, 1, 8, 40)])
def test_chunk_attention_matches_oracle(bits, Hkv, Hq, chunk):
    B = 2
    cfg = bnd.make_config(B, Hkv, Hq, bits, 3000, 4, 32, 16, chunk)
    wl = synth.WORKLOADS["tiny"]
    T = np.stack([synth.key_transform(wl, 7, h).numpy() for h in range(Hkv)])
    t_dev = H.to_dev(T)
    tinv = bnd.compensation(torch.from_numpy(T)).cuda()
    scale = 1 / np.sqrt(128)
    rng = np.random.default_rng(bits * 100 + Hq + chunk)
    gc = bnd.KVCache(cfg)

    def tokens(n):
        x = rng.standard_normal((B, n, Hkv, 128))
        x[..., [9, 99]] *= 15
        return H.to_dev(x.astype(np.float16))

    gc.append(tokens(900), tokens(900), t_dev)  # a bulk prefill before the chunks
    for i, n in enumerate([chunk, 1, max(chunk - 1, 1), chunk, 2 if chunk >= 2 else 1]):
        gc.append(tokens(n), tokens(n), t_dev)
        q = rng.standard_normal((B, n, Hq, 128)).astype(np.float16)
        out = gc.chunk_attn(H.to_dev(q), tinv, scale)
        torch.cuda.synchronize()
        assert gc.status() == 0
        # every counter is back at zero, for the next call of any kind on this workspace
        nt = ticket_words(cfg, B, Hkv)
        assert torch.count_nonzero(gc.workspace[:4 * nt]).item() == 0
        ref = oatt.chunk_decode(H.oracle_cache_from_gpu(gc), q, T, scale)
        H.assert_attention_close(out.cpu().numpy(), ref)
        dec = gc.decode_attn(H.to_dev(q[:, -1]), tinv, scale)  # same workspace, other layout
        torch.cuda.synchronize()
        assert torch.count_nonzero(gc.workspace[:4 * nt]).item() == 0
        if n == 1:
            assert torch.equal(dec, out[:, 0])
        else:  # the chunk's last token sees the whole cache, as a decode of its query does
            H.assert_attention_close(dec.cpu().numpy(), ref[:, -1])


def test_chunk_attention_rejects_oversized_chunk():
    cfg = bnd.make_config(1, 1, 4, 2, 256, 4, 32, 16, 4)
    gc = bnd.KVCache(cfg)
    q = torch.zeros(1, 5, 4, 128, dtype=torch.float16, device="cuda")
    tinv = torch.eye(128, device="cuda")[None].contiguous()
    with pytest.raises(bnd.WushKVError):
        gc.chunk_attn(q, tinv, 0.1)
