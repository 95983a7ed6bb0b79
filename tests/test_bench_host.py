"""Host-side logic of bench.py that needs no GPU: the multi-rank reduction (world size 2
over gloo on CPU), the whole-job throughput, and the algorithmic byte accounting of a
step, checked against the oracle cache's own Algorithm-2 bookkeeping."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
from decode_attention_head_b200 import synth
from oracle import cache as ocache


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r saw device times (r + 1, 10 - r) seconds: the job takes the slowest
        got = bench.max_over_ranks([rank + 1.0, 10.0 - rank], "cpu", world)
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0] == res[1] == [2.0, 10.0]


def test_max_over_ranks_single_process_is_identity():
    assert bench.max_over_ranks([3.0, 4.5], "cpu", 1) == [3.0, 4.5]


def test_job_throughput_counts_every_replica():
    # 4 replicas of 155.4 MB in 25 us (slowest rank): 4 * 6.216 TB/s
    assert bench.job_throughput(4, 155.4e6, 25e-6) == pytest.approx(4 * 6216.0)


@pytest.mark.parametrize("sink,keep,flush", [(4, 32, 16), (0, 8, 1), (4, 128, 16), (2, 5, 7)])
def test_state_mirror_tracks_the_oracle_flush(sink, keep, flush):
    """The byte accounting's (S, S_quant) mirror follows the oracle's Algorithm-2 state
    step for step through decode-style single-token appends."""
    wl = synth.scaled(synth.WORKLOADS["tiny"], batch=1, n_kv_heads=1, n_q_heads=4, s_sink=sink, s_keep=keep,
                      s_flush=flush)
    oc = ocache.Cache(1, 1, 128, 2, 1.0, 99.0, sink, keep, flush, capacity=400, chunk_max=1)
    T = np.eye(128, dtype=np.float16)[None]
    rng = np.random.default_rng(0)
    x = rng.standard_normal((1, 300, 1, 128)).astype(np.float16)
    oc.append(x[:, :100], x[:, :100], T)
    m = bench.StateMirror(wl, int(oc.S[0]), int(oc.S_quant[0]))
    for p in range(100, 300):
        sq_before = int(oc.S_quant[0])
        oc.append(x[:, p:p + 1], x[:, p:p + 1], T)
        nbytes = m.append_bytes(1)
        assert (m.S, m.Sq) == (int(oc.S[0]), int(oc.S_quant[0]))
        nf = int(oc.S_quant[0]) - max(sq_before, sink) if int(oc.S_quant[0]) > sq_before else 0
        assert nbytes == nf * (512 + 2 * 36) + 1024 + 128 * 128 * 2
        nq = max(m.Sq - sink, 0)
        assert m.decode_bytes() == nq * 72 + (m.S - nq) * 512 + 4 * 768 + 128 * 128 * 4


@pytest.mark.parametrize("S0,n", [(300, 170), (100, 33), (37, 500)])
def test_bulk_append_bytes_follow_the_oracle_flush(S0, n):
    """The prefill byte count's flush (positions quantized, ring entries re-read, tokens kept
    fp16) matches the oracle cache's state change on the same bulk append."""
    sink, keep, flush = 4, 32, 16
    wl = synth.scaled(synth.WORKLOADS["tiny"], batch=1, n_kv_heads=1, n_q_heads=4, s_sink=sink, s_keep=keep,
                      s_flush=flush)
    oc = ocache.Cache(1, 1, 128, 2, 1.0, 99.0, sink, keep, flush, capacity=2000, chunk_max=1)
    T = np.eye(128, dtype=np.float16)[None]
    x = np.random.default_rng(1).standard_normal((1, S0 + n, 1, 128)).astype(np.float16)
    for p in range(S0):  # decode-style appends up to S0 (deferred flushes)
        oc.append(x[:, p:p + 1], x[:, p:p + 1], T)
    S, Sq = int(oc.S[0]), int(oc.S_quant[0])
    oc.append(x[:, S0:], x[:, S0:], T)
    lo0 = max(Sq, sink)
    nq = int(oc.S_quant[0]) - lo0 if int(oc.S_quant[0]) > Sq else 0
    from_ring = max(0, min(lo0 + nq, S) - lo0)
    kept = S + n - max(lo0 + nq, S)
    expect = n * 512 + from_ring * 512 + nq * 72 + kept * 512 + 128 * 128 * 2
    assert bench.bulk_append_bytes(wl, S, Sq, n) == expect
    assert int(oc.S[0]) == S + n


@pytest.mark.parametrize("name,expect", [
    ("llama3-8b-layer", 155.4e6), ("qwen3-8b-layer", 76.5e6), ("mha-32l", 74.8e9),
    ("prefill-append-decode", 304.6e6)])
def test_decode_bytes_follow_the_per_unit_costs(name, expect):
    """The roofline's numerator at steady state (S_quant = S - S_keep): per quantized
    token-head (128 * bits / 8 + 4) B for K and again for V, 512 B per fp16 window
    token-head (K and V), 256 B in + 512 B out per query head, 64 KiB of fp32 T_K^{-1} per KV
    head, summed over the workload's layers.  `expect` is that sum to four significant digits."""
    wl = synth.WORKLOADS[name]
    S = wl.context
    got = bench.StateMirror(wl, S, S - wl.s_keep).decode_bytes() * wl.n_layers
    units = wl.batch * wl.n_kv_heads
    nq = S - wl.s_keep - wl.s_sink
    closed = wl.n_layers * (units * (nq * 2 * (128 * wl.bits // 8 + 4) + (wl.s_sink + wl.s_keep) * 512)
                            + wl.batch * wl.n_q_heads * (256 + 512) + wl.n_kv_heads * 128 * 128 * 4)
    assert got == closed
    assert abs(got - expect) <= 5e-4 * expect
