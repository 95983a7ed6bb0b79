"""Writes rms_sigma.txt: fp32 RMS values of fp16 vectors in the fixed summation order of
the QuEST-style quantizer's reading (sigma^2 summed as four runs of 32 consecutive squares,
each run left to right, then (g0 + g1) + (g2 + g3); divided by 128; square root), computed
with a pure-Python IEEE binary32 routine: every operation is done in binary64 and rounded
once to binary32, which for +, *, / and sqrt of binary32 operands gives the correctly
rounded binary32 result (binary64 has more than 2 * 24 + 2 bits).  It uses neither numpy
nor the oracle.

Only vectors on which that order gives a different sigma from each of four other plausible
orders are kept, so a test against this file tells the orders apart:
  l2r     all 128 squares summed left to right;
  seq4    the four runs added as ((g0 + g1) + g2) + g3;
  cross   the four runs added as (g0 + g2) + (g1 + g3);
  runs16  eight runs of 16, added pairwise ((r0+r1)+(r2+r3)) + ((r4+r5)+(r6+r7)).

Run: python tests/golden/make_rms_golden.py   (rewrites rms_sigma.txt beside it)
"""
import math
import os
import random
import struct


def f32(x: float) -> float:
    return struct.unpack("<f", struct.pack("<f", x))[0]


def f16_bits(x: float) -> int:
    return struct.unpack("<H", struct.pack("<e", x))[0]


def f16_value(bits: int) -> float:
    return struct.unpack("<e", struct.pack("<H", bits))[0]


def f32_bits(x: float) -> int:
    return struct.unpack("<I", struct.pack("<f", x))[0]


def run_sum(sq, lo, hi):
    acc = 0.0
    for i in range(lo, hi):
        acc = f32(acc + sq[i])
    return acc


def sigma_from_sum(ss):
    return f32(math.sqrt(f32(ss / 128.0)))


def orders(xs):
    sq = [f32(x * x) for x in xs]
    g = [run_sum(sq, 32 * j, 32 * j + 32) for j in range(4)]
    r = [run_sum(sq, 16 * j, 16 * j + 16) for j in range(8)]
    return {
        "spec": sigma_from_sum(f32(f32(g[0] + g[1]) + f32(g[2] + g[3]))),
        "l2r": sigma_from_sum(run_sum(sq, 0, 128)),
        "seq4": sigma_from_sum(f32(f32(f32(g[0] + g[1]) + g[2]) + g[3])),
        "cross": sigma_from_sum(f32(f32(g[0] + g[2]) + f32(g[1] + g[3]))),
        "runs16": sigma_from_sum(f32(f32(f32(r[0] + r[1]) + f32(r[2] + r[3])) +
                                     f32(f32(r[4] + r[5]) + f32(r[6] + r[7])))),
    }


def main():
    rng = random.Random(20260219)
    rows = []
    tried = 0
    while len(rows) < 12:
        tried += 1
        scale = 10.0 ** rng.uniform(-3.0, 2.5)
        bits = [f16_bits(rng.gauss(0.0, 1.0) * scale * (30.0 if rng.random() < 0.03 else 1.0))
                for _ in range(128)]
        xs = [f16_value(b) for b in bits]
        if any(math.isinf(x) for x in xs):
            continue
        o = orders(xs)
        if all(o["spec"] != o[k] for k in ("l2r", "seq4", "cross", "runs16")):
            rows.append((o, bits))
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "rms_sigma.txt")
    with open(path, "w") as f:
        f.write("# fp32 RMS of fp16 vectors in the order (g0 + g1) + (g2 + g3) of four runs of 32 squares\n")
        f.write("# (\"WUSH-KV: KV Cache Quantization with Data-Adaptive Transforms\", §4.3 / Appendix B.3,\n")
        f.write("# QuEST-style grid scaled by each group's RMS; the summation order is this build's reading).\n")
        f.write("# Written by make_rms_golden.py (pure-Python binary32 arithmetic).  Per line:\n")
        f.write("# sigma_spec sigma_l2r sigma_seq4 sigma_cross sigma_runs16 (fp32 bits, hex), then 128 fp16 bits\n")
        for o, bits in rows:
            head = " ".join(f"{f32_bits(o[k]):08x}" for k in ("spec", "l2r", "seq4", "cross", "runs16"))
            f.write(head + " " + " ".join(f"{b:04x}" for b in bits) + "\n")
    print(f"wrote {len(rows)} vectors ({tried} tried) to {path}")


if __name__ == "__main__":
    main()
