"""Pins for the oracle's weight dequantisation (the DeepSeek-V3 page's BF16 path:
weight_dequant(weight, weight.scale); fp8_cast_bf16.py).

What fixes the expected values:
- with power-of-two scales the product dec(q) * s is exact and fits bf16 (an E4M3 value
  has 4 significant bits), so the output must equal the exact value (Fractions);
- with fp32 scales the output is the fp32 product rounded to bf16: numpy's IEEE fp32
  multiply, then torch's round-to-nearest-even bf16 cast (a library routine);
- block placement: a scale changed in one 128 x 128 block changes only that block;
- round trip: dequant(quant(w)) is within half an FP8 step of w (|w - dq| <= s * ulp/2
  of the code, plus the bf16 rounding), and exact codes map back to themselves.
"""
from fractions import Fraction

import numpy as np
import torch

import oracle as O
import synth


def bf16_bits_of(f32: np.ndarray) -> np.ndarray:
    return torch.from_numpy(f32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def f32_of_bf16(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def test_power_of_two_scales_are_exact():
    rng = np.random.default_rng(1)
    q = rng.integers(0, 256, (256, 384)).astype(np.uint8)
    q[(q & 0x7F) == 0x7F] = 0x10                     # no NaN codes
    s = np.exp2(rng.integers(-20, 20, (2, 3))).astype(np.float32)
    out = O.weight_dequant(q, s)
    for (n, k) in [(0, 0), (5, 200), (130, 10), (255, 383), (200, 300)]:
        exact = Fraction(O.decode(int(q[n, k]))) * Fraction(float(s[n // 128, k // 128]))
        assert Fraction(float(f32_of_bf16(out[n:n + 1, k])[0])) == exact
    dec = np.array([O.decode(c) for c in range(256)], np.float64)
    ref = dec[q] * np.repeat(np.repeat(s.astype(np.float64), 128, 0), 128, 1)
    assert np.array_equal(f32_of_bf16(out).astype(np.float64), ref)


def test_fp32_scales_round_product_then_bf16():
    rng = np.random.default_rng(2)
    q = rng.integers(0, 0x7E, (128, 256)).astype(np.uint8)
    s = rng.uniform(1e-4, 3.0, (1, 2)).astype(np.float32)
    out = O.weight_dequant(q, s)
    dec = np.array([O.decode(c) for c in range(256)], np.float32)
    prod = dec[q] * np.repeat(np.repeat(s, 128, 0), 128, 1)          # IEEE fp32 products
    assert np.array_equal(out, bf16_bits_of(prod))


def test_block_placement_and_per_tensor():
    q = np.full((300, 272), O.encode(2.0), np.uint8)
    s = np.ones((3, 3), np.float32)
    s[1, 2] = 4.0
    out = f32_of_bf16(O.weight_dequant(q, s))
    assert (out[128:256, 256:] == 8.0).all()
    out[128:256, 256:] = 2.0
    assert (out == 2.0).all()
    pt = f32_of_bf16(O.weight_dequant(q, np.array([0.5], np.float32), block=0))
    assert (pt == 1.0).all()


def test_round_trip_bound():
    w = synth.weights(256, 512, 0.02, seed=4)
    q, s = O.weight_quant(w)
    dq = f32_of_bf16(O.weight_dequant(q, s)).astype(np.float64)
    wf = w.float().numpy().astype(np.float64)
    step = np.repeat(np.repeat(s.astype(np.float64), 128, 0), 128, 1)
    # E4M3 relative step 2^-3 near the top of a binade: |w - dq| <= s * 2^-4 * |w/s| + bf16 half ulp
    bound = np.abs(wf) * 2.0 ** -4 + step * 2.0 ** -10 + np.abs(dq) * 2.0 ** -8
    assert (np.abs(wf - dq) <= bound).all()
