"""GPU parity of the delayed-scaling per-tensor quantiser against the oracle's step
function: codes, the clipped-element count, the scale used, and the whole carried
state (next scale, slot index, history) must be bit-exact after every step."""
import numpy as np
import pytest
import torch

import fp8_block_scaled_12_b200 as F
import oracle as O
import synth
from _parity import assert_codes_equal, codes

pytestmark = pytest.mark.gpu

FMTS = [(F.E4M3, O.E4M3, 400.0), (F.E5M2, O.E5M2, 51200.0)]


def compare_state(ds: F.DelayedScaling, st: O.DelayedScalingState, what: str):
    assert ds.scale.cpu().numpy().view(np.uint32)[0] == st.scale.view(np.uint32)[0], f"{what}: next scale"
    assert int(ds.pos.cpu()[0]) == int(st.pos[0]), f"{what}: slot"
    assert np.array_equal(ds.history.cpu().numpy().view(np.uint32), st.history.view(np.uint32)), f"{what}: history"


def run_steps(dev, fmt, algo, hist_len, tensors):
    ds = F.DelayedScaling(hist_len=hist_len, fmt=fmt[0], target=fmt[2], algo=algo, device=dev)
    st = O.DelayedScalingState(hist_len=hist_len)
    oalgo = O.ALGO_MAX if algo == F.AMAX_MAX else O.ALGO_MOST_RECENT
    total_clipped = 0
    for i, x in enumerate(tensors):
        q, s_used, n_clip = ds.step(x.to(dev))
        torch.cuda.synchronize()
        qr, nr, sr = O.delayed_quant(x, st, fmt=fmt[1], target=fmt[2], algo=oalgo)
        assert_codes_equal(codes(q).reshape(-1), qr.reshape(-1), f"step {i} codes")
        assert int(n_clip.cpu()[0]) == nr, f"step {i}: clipped {int(n_clip.cpu()[0])} vs {nr}"
        assert s_used.cpu().numpy().view(np.uint32)[0] == np.float32(sr).view(np.uint32), f"step {i}: scale used"
        compare_state(ds, st, f"step {i}")
        total_clipped += nr
    return total_clipped


@pytest.mark.parametrize("fmt", FMTS, ids=["e4m3", "e5m2"])
@pytest.mark.parametrize("algo", [F.AMAX_MAX, F.AMAX_MOST_RECENT], ids=["max", "most_recent"])
@pytest.mark.parametrize("hist_len", [1, 3, 16])
def test_delayed_steps(cuda_device, fmt, algo, hist_len):
    """Six steps whose spread jumps up and down (so some steps clip, as the page warns
    happens when a step is larger than the previous one), ragged sizes."""
    tensors = []
    for i, (spread, n) in enumerate([(1.0, 4096), (300.0, 8000), (20.0, 2048), (5e4, 65536), (3.0, 8), (0.0, 64)]):
        x = synth.activations(1, n, seed=40 + i, dist="t3").float() * spread
        tensors.append(x.to(torch.bfloat16).reshape(-1))
    clipped = run_steps(cuda_device, fmt, algo, hist_len, tensors)
    assert clipped > 0                  # the sequence does exercise clipping


def test_delayed_boundary_quotients(cuda_device):
    """Quotients exactly at 448 and one fp32 ulp either side, under non-power-of-two
    scales: the carried scale is set directly (the state is the caller's) to
    s0 = fl32(x / 448) and its neighbouring floats, so fl32(x / s) straddles Fmax and
    the clipped count hinges on the quotient's last bit."""
    rng = np.random.default_rng(3)
    xs = (np.array(rng.integers(0x3F80, 0x4480, 16), np.uint32) << 16).view(np.float32)   # bf16 in [1, 1024)
    seen = set()
    for i, xv in enumerate(xs):
        s0 = np.float32(xv) / np.float32(448.0)
        for k in (-2, -1, 0, 1, 2):
            s = (np.array([s0], np.float32).view(np.int32) + np.int32(k)).view(np.float32)[0]
            ds = F.DelayedScaling(hist_len=2, device=cuda_device)
            st = O.DelayedScalingState(hist_len=2)
            ds.scale.fill_(float(s))
            st.scale[0] = s
            x = torch.tensor([float(xv), -float(xv), float(xv) * 0.5] + [0.0] * 5).to(torch.bfloat16)
            q, s_used, n_clip = ds.step(x.to(cuda_device))
            torch.cuda.synchronize()
            qr, nr, sr = O.delayed_quant(x, st)
            assert_codes_equal(codes(q), qr, f"x={xv} s={s} codes")
            assert int(n_clip.cpu()[0]) == nr, f"x={xv} s={s}: clipped {int(n_clip.cpu()[0])} vs {nr}"
            compare_state(ds, st, f"x={xv} s={s}")
            seen.add((np.float32(xv) / s > np.float32(448.0), np.float32(xv) / s == np.float32(448.0)))
    assert len(seen) == 3          # clipped, exactly 448, and just below were all hit


def test_delayed_sweep_size(cuda_device):
    """Sweep tensor 16384 x 7168 (Student-t(3)), three steps with changing spread: state
    and clipped counts exact, codes on every 97th row."""
    dev = cuda_device
    ds = F.DelayedScaling(hist_len=16, device=dev)
    st = O.DelayedScalingState(hist_len=16)
    for i, spread in enumerate([1.0, 40.0, 0.5]):
        x = (synth.activations(16384, 7168, seed=i, dist="t3", device=dev).float() * spread).to(torch.bfloat16)
        q, s_used, n_clip = ds.step(x)
        torch.cuda.synchronize()
        xh = x.cpu()
        # the oracle step on the whole tensor (one C pass over 117 M elements)
        qr, nr, sr = O.delayed_quant(xh, st)
        assert int(n_clip.cpu()[0]) == nr and float(s_used.cpu()[0]) == sr
        compare_state(ds, st, f"sweep step {i}")
        rows = np.arange(0, 16384, 97)
        assert_codes_equal(codes(q)[rows], qr[rows], f"sweep step {i} codes (sampled rows)")
