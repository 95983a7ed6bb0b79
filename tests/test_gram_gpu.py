"""Calibration Gram matrices on the GPU (wushkv_gram_accumulate) against the oracle's
float64 sums, through the C ABI.

Tolerance, from the arithmetic.  A CTA sums at most 4096 tokens of one head on the tensor
cores (tcgen05.mma kind::f16, K = 16 tokens per instruction, fp32 accumulator in tensor
memory); a product of two fp16 values is exact in fp32.  Each MMA adds 16 products to
its fp32 accumulator C.  Aligning the 17 addends to the largest loses at most one fp32 ulp
of it per addend, so one MMA errs by at most 17 * 2^-23 * (|C| + sum |a b|) <= 17 * 2^-23 * A,
with A = sum_t |x_ti| |x_tj| over the CTA's tokens.  Over ceil(T / 16) MMAs that gives
ceil(T / 16) * 17 * 2^-23 * A.  The fp64
atomics add a few 2^-53 A more.
Integer-valued inputs whose partial sums stay below 2^24 are summed exactly, so those
cases are compared bit for bit: they pin every index of the tiling."""
import numpy as np
import pytest
import torch

from decode_attention_head_b200 import binding as bnd
from decode_attention_head_b200 import synth
from oracle import calibration as ocal

pytestmark = pytest.mark.gpu

CTA_TOKENS = 4096


def _gpu_gram(x: np.ndarray, gram: torch.Tensor = None) -> torch.Tensor:
    heads = x.shape[-2]
    g = torch.zeros(heads, 128, 128, dtype=torch.float64, device="cuda") if gram is None else gram
    bnd.gram_accumulate(torch.from_numpy(np.ascontiguousarray(x)).cuda(), g)
    torch.cuda.synchronize()
    return g


def _bound(x: np.ndarray) -> np.ndarray:
    x3 = x.reshape(-1, x.shape[-2], 128)
    a = ocal.gram(np.abs(x3.astype(np.float64)))
    t = min(len(x3), CTA_TOKENS)
    return (-(-t // 16)) * 17 * 2.0 ** -23 * a + 2.0 ** -48 * a


def _check(got: torch.Tensor, x: np.ndarray):
    x3 = x.reshape(-1, x.shape[-2], 128)
    ref = ocal.gram(x3)
    err = np.abs(got.cpu().numpy() - ref)
    bound = _bound(x3)
    assert (err <= bound).all(), f"max err/bound {np.max(err / np.maximum(bound, 1e-300)):.3g}"
    return err, ref


@pytest.mark.parametrize("n", [1, 15, 64, 100, 4096, 4097, 9160])
def test_integer_inputs_bit_exact(n):
    rng = np.random.default_rng(n)
    x = rng.integers(-8, 9, size=(n, 3, 128)).astype(np.float16)  # |partial sums| <= 64 * 4096 < 2^24
    got = _gpu_gram(x).cpu().numpy()
    np.testing.assert_array_equal(got, ocal.gram(x))


@pytest.mark.parametrize("heads,n", [(1, 80000), (3, 50000), (8, 40000)])
def test_integer_inputs_long_runs_bit_exact(heads, n):
    """Runs of 5 to 17 stages of 64 tokens per CTA: every slot of the copy ring is reused."""
    rng = np.random.default_rng(n + heads)
    x = rng.integers(-8, 9, size=(n, heads, 128)).astype(np.float16)  # |partial sums| <= 64 * 4096 < 2^24
    got = _gpu_gram(x).cpu().numpy()
    np.testing.assert_array_equal(got, ocal.gram(x))


def test_single_token_is_exact_outer_product():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((1, 2, 128)) * 3).astype(np.float16)
    got = _gpu_gram(x).cpu().numpy()
    np.testing.assert_array_equal(got, ocal.gram(x))  # one nonzero product per sum


@pytest.mark.parametrize("which", ["k", "v"])
def test_synthetic_keys_and_values_within_bound(which):
    wl = synth.scaled(synth.WORKLOADS["qwen3-8b-layer"], batch=2)
    x = synth.bulk_tokens(wl, 0, 1000, 2600, device="cpu", which=which).numpy()  # [2, 2600, 8, 128]
    got = _gpu_gram(x)
    _check(got, x)
    # (i, j) and (j, i) are one sum each within the bound, so they differ by at most twice it
    g = got.cpu().numpy()
    assert (np.abs(g - np.transpose(g, (0, 2, 1))) <= 2 * _bound(x)).all()


def test_accumulates_across_calls():
    rng = np.random.default_rng(21)
    a = rng.integers(-8, 9, size=(3000, 2, 128)).astype(np.float16)
    b = rng.integers(-8, 9, size=(5000, 2, 128)).astype(np.float16)
    g = _gpu_gram(a)
    _gpu_gram(b, g)
    np.testing.assert_array_equal(g.cpu().numpy(), ocal.gram(np.concatenate([a, b])))
    # zero tokens queue nothing
    before = g.clone()
    bnd.gram_accumulate(torch.empty(0, 2, 128, dtype=torch.float16, device="cuda"), g)
    torch.cuda.synchronize()
    assert torch.equal(g, before)


def test_calibration_sequences_full_size():
    """The configuration bench.py times: four 32,768-token sequences of Qwen3-8B-shaped
    keys (RMSNorm + RoPE) for 8 KV heads, against the oracle over all 131,072 tokens."""
    wl = synth.scaled(synth.WORKLOADS["qwen3-8b-layer"], batch=4)
    xd = synth.bulk_tokens(wl, 0, 0, 32768, device="cuda", which="k")  # [4, 32768, 8, 128]
    g = torch.zeros(8, 128, 128, dtype=torch.float64, device="cuda")
    bnd.gram_accumulate(xd, g)
    torch.cuda.synchronize()
    _check(g, xd.cpu().numpy())
