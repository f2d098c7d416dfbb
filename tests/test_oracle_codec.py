"""Pins for the oracle's FP8 codec against what the pages and mathematics fix.

- Ranges: E4M3 largest finite 448, E5M2 largest finite 57344 ("LLM 推理的 FP8 混合精度
  工程 2026", section 2; "ROCm 7 ... AITER", section 1.1 table).
- E4M3 is the fn variant: no infinity, S.1111.111 is NaN (torch.float8_e4m3fn, named
  in the delayed-scaling listing of the ROCm page, section 4.3).
- Decoding is checked against torch's float8 dtypes (a library routine) for all 256
  codes; encoding against torch's round-to-nearest-even cast inside the finite range,
  plus hand cases for ties, saturation and signed zero.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O

FMTS = [(O.E4M3, torch.float8_e4m3fn, 0x7E, 448.0), (O.E5M2, torch.float8_e5m2, 0x7B, 57344.0)]


@pytest.mark.parametrize("fmt,tdt,top,fmax", FMTS)
def test_decode_all_codes_match_torch(fmt, tdt, top, fmax):
    ref = torch.arange(256, dtype=torch.uint8).view(tdt).to(torch.float64).numpy()
    got = O.decode_table(fmt)
    nan_ref, nan_got = np.isnan(ref), np.isnan(got)
    assert (nan_ref == nan_got).all()
    assert (ref[~nan_ref] == got[~nan_got]).all()
    # signed zero for 0x80
    assert math.copysign(1.0, got[0x80]) == -1.0


def test_e4m3_closed_form_pins():
    assert O.fmax(O.E4M3) == 448.0
    assert O.decode(0x7E) == 448.0 and O.decode(0xFE) == -448.0
    assert O.decode(0x01) == 2.0 ** -9          # smallest subnormal
    assert O.decode(0x08) == 2.0 ** -6          # smallest normal
    assert O.decode(0x07) == 7 * 2.0 ** -9      # largest subnormal
    assert O.decode(0x38) == 1.0                # exponent field 7 = bias
    assert math.isnan(O.decode(0x7F)) and math.isnan(O.decode(0xFF))
    vals = O.decode_table(O.E4M3)
    assert not np.isinf(vals).any()             # e4m3fn has no infinity
    assert np.isnan(vals).sum() == 2


def test_e5m2_closed_form_pins():
    assert O.fmax(O.E5M2) == 57344.0
    assert O.decode(0x7B, O.E5M2) == 57344.0
    assert O.decode(0x7C, O.E5M2) == math.inf and O.decode(0xFC, O.E5M2) == -math.inf
    assert O.decode(0x01, O.E5M2) == 2.0 ** -16
    assert O.decode(0x04, O.E5M2) == 2.0 ** -14
    assert O.decode(0x3C, O.E5M2) == 1.0
    vals = O.decode_table(O.E5M2)
    assert np.isnan(vals).sum() == 6


@pytest.mark.parametrize("fmt,tdt,top,fmax", FMTS)
def test_encode_roundtrip_every_code(fmt, tdt, top, fmax):
    for c in range(256):
        v = O.decode(c, fmt)
        if math.isnan(v) or math.isinf(v):
            continue
        assert O.encode(np.float32(v), fmt) == c, hex(c)


def _ulp_step(v, direction):
    return float(np.nextafter(np.float32(v), np.float32(direction)))


@pytest.mark.parametrize("fmt,tdt,top,fmax", FMTS)
def test_midpoints_round_to_even_and_neighbours_to_nearest(fmt, tdt, top, fmax):
    for c in range(0, top):
        lo, hi = O.decode(c, fmt), O.decode(c + 1, fmt)
        mid = (lo + hi) / 2.0
        assert float(np.float32(mid)) == mid      # every midpoint is an fp32 value
        even = c if c % 2 == 0 else c + 1
        assert O.encode(np.float32(mid), fmt) == even
        assert O.encode(np.float32(_ulp_step(mid, -1)), fmt) == c
        assert O.encode(np.float32(_ulp_step(mid, 1e30)), fmt) == c + 1
        # negative side mirrors with the sign bit
        assert O.encode(np.float32(-mid), fmt) == 0x80 | even


def test_saturation_e4m3():
    for v in [448.0, 448.5, 463.9, 464.0, 480.0, 1e30, math.inf, 3.0e38]:
        assert O.encode(v) == 0x7E, v
        assert O.encode(-v) == 0xFE, v


def test_saturation_e5m2():
    for v in [57344.0, 57344.0 * 1.07, 61439.0, 61440.0, 1e30, math.inf]:
        assert O.encode(v, O.E5M2) == 0x7B, v
        assert O.encode(-v, O.E5M2) == 0xFB, v


def test_signed_zero_and_underflow():
    assert O.encode(0.0) == 0x00
    assert O.encode(-0.0) == 0x80
    assert O.encode(-1e-30) == 0x80
    assert O.encode(2.0 ** -10) == 0x00          # exact tie between 0 and 2^-9 -> even (0)
    assert O.encode(np.float32(2.0 ** -10 * 1.0000001)) == 0x01
    assert O.encode(3 * 2.0 ** -10) == 0x02      # tie between 1 and 2 (x 2^-9) -> even
    assert O.encode(2.0 ** -17, O.E5M2) == 0x00  # tie at half the smallest e5m2 subnormal
    assert O.encode(math.nan) == 0x7F


@pytest.mark.parametrize("fmt,tdt,top,fmax", FMTS)
def test_encode_agrees_with_torch_cast_inside_range(fmt, tdt, top, fmax):
    """torch's fp32 -> float8 cast is round-to-nearest-even; inside (-Fmax, Fmax) no
    saturation rule is involved, so it must agree with the oracle exactly."""
    rng = np.random.default_rng(1234)
    # (a) every bf16 value inside the range, (b) random fp32 with exponents across the range
    bf = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    bf = bf[np.isfinite(bf) & (np.abs(bf) < fmax)]
    e = rng.uniform(-24 if fmt == O.E4M3 else -32, math.log2(fmax), 60000)
    r = (rng.choice([-1.0, 1.0], e.size) * np.exp2(e)).astype(np.float32)
    r = r[np.abs(r) < fmax]
    for arr in (bf, r):
        ref = torch.from_numpy(arr.copy()).to(tdt).view(torch.uint8).numpy()
        got = np.array([O.encode(float(v), fmt) for v in arr], dtype=np.uint8)
        bad = np.nonzero(ref != got)[0]
        assert bad.size == 0, (arr[bad[:5]], ref[bad[:5]], got[bad[:5]])
