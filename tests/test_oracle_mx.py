"""Pins for the oracle's MXFP8 functions (E8M0 exponent bytes, 32-element block
quantisation, GEMM with per-32-element scales on both operands).

What fixes the expected values:
- an E8M0 byte b is the power of two 2^(b-127), 0xFF is NaN (8 exponent bits, no sign,
  no mantissa: "ROCm 7 ... AITER", section 1.1 lists MXFP8 as 8 bits plus a shared
  exponent) -- checked against math.ldexp;
- blocks are 32 consecutive elements of a row, each with its own scale (same page,
  section 1.2): an outlier planted in one block moves only that block's byte, and a
  ragged last block covers only the valid elements;
- the shared exponent follows the reading recorded for the oracle: the smallest power
  of two s = 2^e (e >= -126) with amax / Fmax <= s, checked with exact rationals;
- codes: the value nearest to x / s, brute-forced over all 256 codes with Fractions;
- GEMM: exact integer dot products per 32-element block times exact powers of two
  (Python integers / Fractions), and a hand-derived two-block case.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O
import synth
from test_oracle_quant import nearest_code_bruteforce


def exact_e(amax: Fraction, fmax: float) -> int:
    """Smallest e >= -126 with amax / fmax <= 2^e, by exact rational arithmetic."""
    t = amax / Fraction(fmax)
    e = -126
    while Fraction(2) ** e < t:
        e += 1
    return e


def test_e8m0_decode_closed_form():
    for b in range(255):
        assert O.e8m0_decode(b) == math.ldexp(1.0, b - 127)
    assert math.isnan(O.e8m0_decode(0xFF))
    assert O.e8m0_decode(127) == 1.0 and O.e8m0_decode(0) == 2.0 ** -127 and O.e8m0_decode(254) == 2.0 ** 127


@pytest.mark.parametrize("fmt", [O.E4M3, O.E5M2], ids=["e4m3", "e5m2"])
def test_mx_quant_bruteforce(fmt):
    """Tiny Student-t input with planted outliers: every byte by exact rationals, every
    code by scanning all codes."""
    x = synth.activations(3, 96, seed=5, dist="t3")
    x[1, 40] = 300.0
    x[2, 65] = -7000.0
    q, e8 = O.mx_quant(x, fmt=fmt)
    assert e8.shape == (3, 3)
    xf = x.float().numpy()
    fmax = O.fmax(fmt)
    for m in range(3):
        for g in range(3):
            blk = xf[m, 32 * g:32 * g + 32]
            amax = max(Fraction(float(abs(v))) for v in blk)
            e = exact_e(amax, fmax)
            assert e8[m, g] == e + 127, (m, g)
            s = np.float32(2.0 ** e)
            for k in range(32):
                t = np.float32(blk[k]) / s
                assert q[m, 32 * g + k] == nearest_code_bruteforce(t, fmt), (m, g, k)


def test_mx_block_boundaries_and_placement():
    """448 in a block gives byte 127 (s = 1); 450 gives 128; an all-zero block gives
    the floor 2^-126 (byte 1); a planted outlier changes only its own block's byte;
    a ragged last block (K = 48: blocks of 32 and 16) ignores the missing elements."""
    x = torch.zeros(4, 48, dtype=torch.bfloat16)
    x[0, :32] = 1.0
    x[0, 5] = 448.0
    x[1, 32:] = -450.0                       # bf16 has no 449; 450 > 448 needs s = 2
    x[2, 3] = 1.0
    base_q, base_e = O.mx_quant(x)
    assert base_e[0, 0] == 127 and base_e[1, 1] == 128 and base_e[3, 0] == 1 and base_e[3, 1] == 1
    assert base_q[0, 5] == 0x7E and base_q[0, 0] == O.encode(1.0)
    x2 = x.clone()
    x2[2, 40] = 1000.0                        # row 2, block 1 only
    q2, e2 = O.mx_quant(x2)
    changed = np.argwhere(e2 != base_e)
    assert changed.tolist() == [[2, 1]]
    assert (q2[:, :32] == base_q[:, :32]).all() and (q2[[0, 1, 3]] == base_q[[0, 1, 3]]).all()


def test_mx_gemm_hand_case():
    """K = 64, one row each: a = 1.0 (block 0) and 2.0 (block 1); w = 1.0; exponent
    bytes ea = (127, 130) -> (1, 8) and ew = (126, 127) -> (0.5, 1):
    y = 32 * (1 * 1) * (1 * 0.5) + 32 * (2 * 8) * (1 * 1) = 16 + 512 = 528."""
    one, two = O.encode(1.0), O.encode(2.0)
    qa = np.array([[one] * 32 + [two] * 32], np.uint8)
    qw = np.array([[one] * 64], np.uint8)
    ea = np.array([[127, 130]], np.uint8)
    ew = np.array([[126, 127]], np.uint8)
    y, b = O.mx_gemm_rows(qa, ea, qw, ew)
    assert y[0, 0] == 528.0 and b[0, 0] == 528.0


def test_mx_gemm_integer_blocks_exact():
    """Small-integer codes with random per-block exponents: y equals the exact sum over
    blocks of 2^(ea + ew - 254) * (integer dot product of the block)."""
    rng = np.random.default_rng(3)
    M, N, K = 5, 7, 160
    A = rng.integers(-8, 9, (M, K))
    W = rng.integers(-8, 9, (N, K))
    qa = torch.from_numpy(A.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    qw = torch.from_numpy(W.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ea = rng.integers(120, 135, (M, K // 32)).astype(np.uint8)
    ew = rng.integers(120, 135, (N, K // 32)).astype(np.uint8)
    y, bound = O.mx_gemm_rows(qa, ea, qw, ew)
    for m in range(M):
        for n in range(N):
            ref = Fraction(0)
            for g in range(K // 32):
                dot = int(np.dot(A[m, 32 * g:32 * g + 32], W[n, 32 * g:32 * g + 32]))
                ref += dot * Fraction(2) ** (int(ea[m, g]) + int(ew[n, g]) - 254)
            assert Fraction(y[m, n]) == ref, (m, n)
    assert (bound >= np.abs(y)).all()

