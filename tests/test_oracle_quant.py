"""Pins for the oracle's quantisers (act_quant per token per 128 channels, 128x128
weight blocks, per-tensor e4m3 / e5m2).

What fixes the expected values:
- scale = amax / Fmax ("FP8 推理", Dynamic Scaling; Fmax 448 / 57344 from the FP8
  engineering page, section 2), checked with numpy's IEEE fp32 division;
- ue8m0 ("DeepSeek-V3 在 AMD MI250", key config table) = the power of two at or above
  amax/448, checked with exact rational arithmetic;
- FP8Cast(x / s) ("量化：FP8 与混合精度推理", FP8 也需要 scale): each code is the value
  nearest to fl32(x / s), brute-forced over all 256 codes with Fractions on tiny inputs;
- block / group placement: an outlier planted in one block moves only that block's
  scale (catches transposed or shifted indices).
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O
import synth


def bf16(a):
    return torch.tensor(a, dtype=torch.float32).to(torch.bfloat16)


def bits_to_f32(x_bf16):
    return x_bf16.to(torch.float32).numpy()


def nearest_code_bruteforce(t: np.float32, fmt=O.E4M3):
    """Nearest code to the fp32 value t by scanning every code (ties -> even mantissa,
    beyond the largest finite value -> saturate)."""
    fmax = O.fmax(fmt)
    tv = Fraction(float(t))
    if abs(tv) >= Fraction(fmax):
        return (0x80 if t < 0 or (t == 0 and np.signbit(t)) else 0) | (0x7E if fmt == O.E4M3 else 0x7B)
    best, bestd = None, None
    for c in range(128):
        v = O.decode(c, fmt)
        if not np.isfinite(v):
            continue
        d = abs(Fraction(v) - abs(tv))
        if bestd is None or d < bestd or (d == bestd and (c & 1) == 0):
            best, bestd = c, d
    return best | (0x80 if np.signbit(t) else 0)


def test_scale_formula_fp32_matches_ieee_division():
    rng = np.random.default_rng(7)
    amax = np.abs(rng.standard_normal(2000).astype(np.float32)) * np.float32(37.0)
    for a in amax:
        a_bf = np.float32(bf16(float(a)).item())
        s = O.scale_from_amax(float(a_bf), O.E4M3, O.SCALE_FP32)
        assert s == np.float32(a_bf) / np.float32(448.0)
        s5 = O.scale_from_amax(float(a_bf), O.E5M2, O.SCALE_FP32)
        assert s5 == np.float32(a_bf) / np.float32(57344.0)


def test_scale_formula_ue8m0_is_power_of_two_at_or_above():
    rng = np.random.default_rng(8)
    for a in np.abs(rng.standard_normal(2000).astype(np.float32)) * np.float32(1000.0):
        a = float(np.float32(bf16(float(a)).item()))
        if a == 0.0:
            continue
        s = O.scale_from_amax(a, O.E4M3, O.SCALE_UE8M0)
        m, e = np.frexp(s)
        assert m == 0.5                                   # a power of two
        q = Fraction(float(np.float32(a) / np.float32(448.0)))
        assert Fraction(s) / 2 < q <= Fraction(s)
    assert O.scale_from_amax(448.0, O.E4M3, O.SCALE_UE8M0) == 1.0
    assert O.scale_from_amax(449.0, O.E4M3, O.SCALE_UE8M0) == 2.0
    assert O.scale_from_amax(224.0, O.E4M3, O.SCALE_UE8M0) == 0.5


def test_zero_group_scale_floor():
    for sf in (O.SCALE_FP32, O.SCALE_UE8M0):
        assert O.scale_from_amax(0.0, O.E4M3, sf) == 2.0 ** -126
    x = torch.zeros(2, 128, dtype=torch.bfloat16)
    x[1] = -0.0
    q, s = O.act_quant(x)
    assert (s == np.float32(2.0 ** -126)).all()
    assert (q[0] == 0x00).all() and (q[1] == 0x80).all()


def test_group_amax_448_gives_unit_scale_and_plain_codes():
    rng = np.random.default_rng(3)
    v = rng.uniform(-440, 440, 128).astype(np.float32)
    v[17] = 448.0
    x = bf16(v).reshape(1, 128)
    for sf in (O.SCALE_FP32, O.SCALE_UE8M0):
        q, s = O.act_quant(x, scale_fmt=sf)
        assert s[0, 0] == 1.0
        xs = bits_to_f32(x)[0]
        assert all(q[0, k] == O.encode(float(xs[k])) for k in range(128))


def test_outlier_maps_to_max_code_and_codes_are_nearest():
    """Tiny brute force: one x20 outlier per group; every code is the nearest value to
    fl32(x / s); the outlier lands on +-448 (fp32 scales)."""
    x = synth.activations(4, 256, seed=11, outliers=[5, 200], factor=20.0)
    xs = bits_to_f32(x)
    for sf in (O.SCALE_FP32, O.SCALE_UE8M0):
        q, s = O.act_quant(x, scale_fmt=sf)
        assert s.shape == (4, 2)
        for m in range(4):
            for g in range(2):
                grp = xs[m, g * 128:(g + 1) * 128]
                amax = np.float32(np.abs(grp).max())
                assert s[m, g] == O.scale_from_amax(float(amax), O.E4M3, sf)
                for k in range(128):
                    t = np.float32(grp[k]) / np.float32(s[m, g])
                    assert q[m, g * 128 + k] == nearest_code_bruteforce(t), (m, g, k)
                if sf == O.SCALE_FP32:
                    kmax = int(np.argmax(np.abs(grp)))
                    assert q[m, g * 128 + kmax] & 0x7F == 0x7E


def test_dequantised_values_bounded():
    """fp32 scales: |dec(q) * s| <= amax (up to the rounding of s).  Both formats: the
    code is within half an E4M3 spacing of x / s (relative 2^-4 in the normal range,
    absolute 2^-10 below 2^-6) -- before the division's own fp32 rounding."""
    x = synth.activations(8, 384, seed=5, dist="t3")
    xs = bits_to_f32(x).astype(np.float64)
    table = O.decode_table()
    for sf in (O.SCALE_FP32, O.SCALE_UE8M0):
        q, s = O.act_quant(x, scale_fmt=sf)
        srep = np.repeat(s.astype(np.float64), 128, axis=1)
        deq = table[q] * srep
        if sf == O.SCALE_FP32:
            amax = np.repeat(np.abs(xs).reshape(8, 3, 128).max(axis=2), 128, axis=1)
            assert (np.abs(deq) <= amax * (1 + 2.0 ** -23)).all()
        t = xs / srep
        err = np.abs(table[q] - t)
        allowed = np.maximum(np.abs(t) * 2.0 ** -4, 2.0 ** -10) * (1 + 2.0 ** -20)
        assert (err <= allowed).all()


def test_ragged_last_group_uses_valid_elements_only():
    K = 200                                          # groups of 128 and 72
    x = synth.activations(3, K, seed=2)
    xs = bits_to_f32(x)
    q, s = O.act_quant(x)
    assert s.shape == (3, 2)
    for m in range(3):
        assert s[m, 1] == np.float32(np.abs(xs[m, 128:]).max()) / np.float32(448.0)
        assert s[m, 0] == np.float32(np.abs(xs[m, :128]).max()) / np.float32(448.0)


def test_weight_block_placement():
    """An outlier planted in block (1, 2) raises only that block's scale."""
    w = synth.weights(256, 384, 0.02, seed=4)
    q0, s0 = O.weight_quant(w)
    assert s0.shape == (2, 3)
    w2 = w.clone()
    w2[128 + 9, 256 + 77] = 50.0
    q1, s1 = O.weight_quant(w2)
    diff = s1 != s0
    assert diff[1, 2] and diff.sum() == 1
    assert s1[1, 2] == np.float32(bf16(50.0).item()) / np.float32(448.0)
    assert q1[128 + 9, 256 + 77] == 0x7E
    # codes outside the block are unchanged
    mask = np.ones_like(q0, dtype=bool)
    mask[128:256, 256:384] = False
    assert (q0[mask] == q1[mask]).all()


def test_weight_block_scale_is_block_amax():
    w = synth.weights(300, 260, 0.05, seed=9)        # ragged in both dimensions
    ws = bits_to_f32(w)
    for sf in (O.SCALE_FP32, O.SCALE_UE8M0):
        q, s = O.weight_quant(w, scale_fmt=sf)
        assert s.shape == (3, 3)
        for bn in range(3):
            for bk in range(3):
                blk = ws[bn * 128:(bn + 1) * 128, bk * 128:(bk + 1) * 128]
                assert s[bn, bk] == O.scale_from_amax(float(np.abs(blk).max()), O.E4M3, sf)


@pytest.mark.parametrize("fmt,top,fmax", [(O.E4M3, 0x7E, 448.0), (O.E5M2, 0x7B, 57344.0)])
def test_per_tensor(fmt, top, fmax):
    x = synth.activations(64, 256, seed=6, dist="t3")
    xs = bits_to_f32(x)
    q, s = O.tensor_quant(x, fmt=fmt)
    amax = np.float32(np.abs(xs).max())
    assert s[0] == amax / np.float32(fmax)
    i = np.unravel_index(np.argmax(np.abs(xs)), xs.shape)
    assert q[i] & 0x7F == top
    # a sample of codes against the brute-force nearest value
    rng = np.random.default_rng(0)
    for _ in range(300):
        r, c = rng.integers(0, 64), rng.integers(0, 256)
        t = np.float32(xs[r, c]) / np.float32(s[0])
        assert q[r, c] == nearest_code_bruteforce(t, fmt)
    # the weight_quant(block=0) entry is the same per-tensor rule
    q2, s2 = O.weight_quant(x, block=0, fmt=fmt)
    assert (q2 == q).all() and s2[0] == s[0]
