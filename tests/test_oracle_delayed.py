"""Pins for the oracle's delayed-scaling step (the ROCm/AITER page, section 4.3: divide
by the previous step's scale, clamp to +-448, cast to float8_e4m3fn, then next scale =
amax / 400 starting from 1.0; section 6: an amax history whose max sets the scale; the
checklist's clipped-element rate).

What fixes the expected values:
- a three-step sequence worked by hand (scales, clip counts, history ring, slot
  clearing) for both history rules;
- codes: the value nearest to fl32(x / s_prev) (numpy's IEEE division), brute-forced
  over all codes; clip counts: numpy's count of |fl32(x / s_prev)| > Fmax;
- the zero-amax floor 2^-126 and the E5M2 range.
"""
import numpy as np
import pytest
import torch

import oracle as O
from test_oracle_quant import nearest_code_bruteforce


def t(vals, n=64):
    a = np.zeros(n, np.float32)
    a[:len(vals)] = vals
    return torch.from_numpy(a).to(torch.bfloat16)


def test_hand_sequence_history_max():
    st = O.DelayedScalingState(hist_len=2)
    # step 1: previous scale 1.0 (the page's initial value); 800 and -500 exceed 448
    q, nclip, s_used = O.delayed_quant(t([800.0, -500.0, 100.0, 1.0]), st)
    assert s_used == 1.0 and nclip == 2
    assert q[0] == 0x7E and q[1] == 0xFE             # clamped to +-448
    assert list(st.history) == [800.0, 0.0] and st.pos[0] == 1
    assert st.scale[0] == 2.0                        # 800 / 400
    # step 2: amax 100, scale 2 from step 1; the history max is still 800
    q, nclip, s_used = O.delayed_quant(t([100.0, -3.0]), st)
    assert s_used == 2.0 and nclip == 0
    assert q[0] == O.encode(50.0) and q[1] == O.encode(-1.5)
    assert list(st.history) == [0.0, 100.0] and st.pos[0] == 0     # slot 0 cleared for step 3
    assert st.scale[0] == 2.0
    # step 3: the history now holds 100 twice -> 100 / 400
    q, nclip, s_used = O.delayed_quant(t([100.0]), st)
    assert s_used == 2.0 and nclip == 0
    assert list(st.history) == [100.0, 0.0] and st.pos[0] == 1
    assert st.scale[0] == 0.25


def test_hand_sequence_most_recent():
    st = O.DelayedScalingState(hist_len=4)
    O.delayed_quant(t([800.0]), st, algo=O.ALGO_MOST_RECENT)
    assert st.scale[0] == 2.0
    q, nclip, s_used = O.delayed_quant(t([100.0, 1000.0]), st, algo=O.ALGO_MOST_RECENT)
    assert s_used == 2.0 and nclip == 1              # 1000 / 2 = 500 > 448
    assert st.scale[0] == 2.5                        # 1000 / 400 (the most recent amax)
    O.delayed_quant(t([40.0]), st, algo=O.ALGO_MOST_RECENT)
    assert st.scale[0] == np.float32(40.0) / np.float32(400.0)     # fl32(40 / 400)


def test_zero_tensor_floors_the_scale():
    st = O.DelayedScalingState(hist_len=1)
    q, nclip, s_used = O.delayed_quant(t([]), st)
    assert nclip == 0 and (q == 0).all()
    assert st.scale[0] == np.float32(2.0 ** -126)
    assert list(st.history) == [0.0] and st.pos[0] == 0


@pytest.mark.parametrize("fmt", [O.E4M3, O.E5M2], ids=["e4m3", "e5m2"])
def test_codes_and_clip_counts_bruteforce(fmt):
    """Four steps of Student-t tensors whose spread grows and shrinks, so some steps
    clip: codes against a scan of all codes, clip counts against numpy."""
    rng = np.random.default_rng(12)
    fmax = O.fmax(fmt)
    target = 400.0 if fmt == O.E4M3 else 51200.0
    st = O.DelayedScalingState(hist_len=3)
    for step, spread in enumerate([3.0, 300.0, 20.0, 5e4]):
        xf = (rng.standard_t(3, 96) * spread).astype(np.float32)
        x = torch.from_numpy(xf).to(torch.bfloat16)
        xv = x.float().numpy()
        s_prev = np.float32(st.scale[0])
        q, nclip, s_used = O.delayed_quant(x, st, fmt=fmt, target=target)
        assert np.float32(s_used) == s_prev
        quot = xv / s_prev
        assert nclip == int((np.abs(quot) > fmax).sum()), step
        for i in range(96):
            assert q[i] == nearest_code_bruteforce(np.float32(quot[i]), fmt), (step, i)
        amax_hist = np.float32(st.history.max())
        assert st.scale[0] == max(amax_hist / np.float32(target), np.float32(2.0 ** -126))
