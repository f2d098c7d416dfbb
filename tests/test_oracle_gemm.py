"""Pins for the oracle's block-scaled GEMM and grouped GEMM.

- A hand-computed 2x2x256 case with two K-blocks and different scales
  (tests/golden/tiny_gemm_hand.json, derivation inside).
- Special cases that reduce to a library routine: with small-integer codes every
  product and partial sum is exact, so y equals numpy's int64 matmul (all scales 1)
  or a per-block int64 matmul times the power-of-two scales.
- The grouped GEMM on expert-sorted rows equals the per-expert integer matmul; rows
  outside every group are zero; empty groups are skipped.
- bf16 rounding of the fp64 result: exact values stay, midpoints go to even.
"""
import json
import os

import numpy as np
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "tiny_gemm_hand.json")

# E4M3 codes of the small integers -8..8 (exact values), built from the codec
INT_CODE = {}
for c in range(256):
    v = O.decode(c)
    if np.isfinite(v) and float(v).is_integer() and -8 <= v <= 8 and not (v == 0 and c == 0x80):
        INT_CODE[int(v)] = c


def int_codes(vals):
    return np.vectorize(lambda v: INT_CODE[int(v)])(vals).astype(np.uint8)


def test_hand_computed_tiny_case():
    g = json.load(open(GOLDEN))
    M, N, K = g["M"], g["N"], g["K"]
    qa = np.zeros((M, K), np.uint8)
    qa[0, :128], qa[0, 128:] = 0x38, 0x40
    qa[1, 0:128:2], qa[1, 1:128:2] = 0xB8, 0x30
    qa[1, 128:160], qa[1, 160:] = 0x44, 0x00
    qw = np.zeros((N, K), np.uint8)
    qw[0, :] = 0x38
    qw[1, :64], qw[1, 64:] = 0x48, 0xC0
    sa = np.array(g["sa"], np.float32)
    sw = np.array(g["sw"], np.float32)
    y, b = O.gemm_rows(qa, sa, qw, sw)
    assert (y == np.array(g["y"])).all(), y
    assert (b == np.array(g["bound"])).all(), b


def test_integer_codes_unit_scales_equal_int_matmul():
    rng = np.random.default_rng(21)
    M, N, K = 5, 40, 512
    A = rng.integers(-8, 9, (M, K))
    W = rng.integers(-8, 9, (N, K))
    y, b = O.gemm_rows(int_codes(A), np.ones((M, K // 128), np.float32),
                       int_codes(W), np.ones((1, K // 128), np.float32))
    assert (y == (A @ W.T).astype(np.float64)).all()
    assert (b == (np.abs(A) @ np.abs(W).T).astype(np.float64)).all()


def test_block_scales_are_placed_per_row_kblock_and_nblock():
    rng = np.random.default_rng(22)
    M, N, K = 3, 256, 384                     # 2 weight row-blocks, 3 K-blocks
    A = rng.integers(-8, 9, (M, K))
    W = rng.integers(-8, 9, (N, K))
    sa = np.exp2(rng.integers(-4, 5, (M, 3))).astype(np.float32)
    sw = np.exp2(rng.integers(-4, 5, (2, 3))).astype(np.float32)
    y, _ = O.gemm_rows(int_codes(A), sa, int_codes(W), sw)
    ref = np.zeros((M, N))
    for kb in range(3):
        part = A[:, kb * 128:(kb + 1) * 128] @ W[:, kb * 128:(kb + 1) * 128].T
        ref += sa[:, kb:kb + 1].astype(np.float64) * np.repeat(sw[:, kb], 128)[None, :] * part
    assert (y == ref).all()
    # a row subset gives the same rows
    y2, _ = O.gemm_rows(int_codes(A), sa, int_codes(W), sw, rows=[2, 0])
    assert (y2 == ref[[2, 0]]).all()


def test_grouped_rows_follow_their_expert():
    rng = np.random.default_rng(23)
    E, N, K = 3, 128, 256
    off = np.array([0, 2, 2, 5], np.int32)     # expert 1 is empty
    A = rng.integers(-8, 9, (6, K))           # row 5 lies outside every group
    W = rng.integers(-8, 9, (E, N, K))
    sa = np.ones((6, 2), np.float32)
    sw = np.exp2(rng.integers(-2, 3, (E, 1, 2))).astype(np.float32)
    y, _ = O.grouped_gemm_rows(int_codes(A), sa, int_codes(W.reshape(E * N, K)).reshape(E, N, K),
                               sw, off, rows=np.arange(6))
    for r in range(6):
        e = 0 if r < 2 else (2 if r < 5 else None)
        if e is None:
            assert (y[r] == 0).all()
            continue
        ref = sum(sw[e, 0, kb] * (A[r, kb * 128:(kb + 1) * 128] @ W[e, :, kb * 128:(kb + 1) * 128].T)
                  for kb in range(2))
        assert (y[r] == ref).all()


def test_round_bf16_direct():
    # exact bf16 values are unchanged; compare bit patterns with torch's fp32 -> bf16 cast
    vals = np.array([1.0, -2.5, 3.0e38, 1.0e-40, 0.0, -0.0, 448.0, 1.0 / 3.0], np.float64)
    exact = torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16)
    ex_bits = exact.view(torch.int16).numpy().view(np.uint16)
    back = exact.to(torch.float64).numpy()
    assert (O.round_bf16(back) == ex_bits).all()
    # midpoints between adjacent bf16 values go to the even pattern; +-tiny goes to nearest
    for base in [1.0, 1.0078125, 3.5, 1e-3, 2.0 ** -130]:
        b0 = torch.tensor([base], dtype=torch.float32).to(torch.bfloat16).view(torch.int16).item() & 0xFFFF
        lo = float(torch.tensor([b0], dtype=torch.int16).view(torch.bfloat16).item())
        hi = float(torch.tensor([b0 + 1], dtype=torch.int16).view(torch.bfloat16).item())
        mid = (lo + hi) / 2
        even = b0 if b0 % 2 == 0 else b0 + 1
        assert O.round_bf16(np.array([mid]))[0] == even
        assert O.round_bf16(np.array([mid - (hi - lo) * 2 ** -30]))[0] == b0
        assert O.round_bf16(np.array([mid + (hi - lo) * 2 ** -30]))[0] == b0 + 1
    # values with <= 24 significant bits: torch's fp32 -> bf16 cast is a single rounding
    rng = np.random.default_rng(5)
    f = rng.standard_normal(5000).astype(np.float32)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert (O.round_bf16(f.astype(np.float64)) == ref).all()
