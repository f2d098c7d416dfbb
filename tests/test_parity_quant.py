"""GPU parity of the quantisers against the CPU oracle: codes and scales must be
bit-exact.  Inputs come from the seeded generator (synth) or are built here to hit
rounding boundaries; the oracle always sees the same bf16 bytes as the GPU."""
import numpy as np
import pytest
import torch

import fp8_block_scaled_12_b200 as F
import oracle as O
import synth
from _parity import THREADS, assert_codes_equal, assert_scales_equal, codes

pytestmark = pytest.mark.gpu

FMTS = [(F.E4M3, O.E4M3), (F.E5M2, O.E5M2)]
SFS = [(F.SCALE_FP32, O.SCALE_FP32), (F.SCALE_UE8M0, O.SCALE_UE8M0)]


def run_act(x_cpu, fmt, sf, dev, ldx=None):
    M, K = x_cpu.shape
    if ldx is None:
        xd = x_cpu.to(dev)
    else:
        buf = torch.zeros((M, ldx), dtype=torch.bfloat16, device=dev)
        buf[:, :K] = x_cpu.to(dev)
        xd = buf[:, :K]
    q, s = F.act_quant(xd, fmt=fmt, scale_fmt=sf)
    torch.cuda.synchronize()
    return codes(q), s.cpu().numpy()


@pytest.mark.parametrize("fmt", FMTS, ids=["e4m3", "e5m2"])
@pytest.mark.parametrize("sf", SFS, ids=["fp32", "ue8m0"])
def test_act_quant_tiny_config(cuda_device, fmt, sf):
    p = synth.TINY.params
    x = synth.activations(p["M"], p["K"], seed=0, outliers=p["outliers"], factor=p["factor"])
    q, s = run_act(x, fmt[0], sf[0], cuda_device)
    qr, sr = O.act_quant(x, fmt=fmt[1], scale_fmt=sf[1])
    assert_codes_equal(q, qr, "codes")
    assert_scales_equal(s, sr, "scales")


@pytest.mark.parametrize("shape", [(1, 16), (37, 208), (5, 7168), (129, 4112), (1000, 1040)])
@pytest.mark.parametrize("sf", SFS, ids=["fp32", "ue8m0"])
def test_act_quant_ragged_shapes(cuda_device, shape, sf):
    M, K = shape
    x = synth.activations(M, K, seed=3, dist="t3")
    q, s = run_act(x, F.E4M3, sf[0], cuda_device)
    qr, sr = O.act_quant(x, scale_fmt=sf[1])
    assert_codes_equal(q, qr, f"codes {shape}")
    assert_scales_equal(s, sr, f"scales {shape}")


def test_act_quant_row_stride(cuda_device):
    x = synth.activations(33, 384, seed=4, outliers=[1, 200], factor=30.0)
    q, s = run_act(x, F.E4M3, F.SCALE_FP32, cuda_device, ldx=392)
    qr, sr = O.act_quant(x)
    assert_codes_equal(q, qr, "codes")
    assert_scales_equal(s, sr, "scales")


def _boundary_rows():
    """Rows of 128 bf16 values: each row holds one amax value and 127 values drawn from
    every positive / negative bf16 value up to that amax, so x / s sweeps all
    magnitudes (rounding ties, the subnormal range, signed zeros, values that round up
    to Fmax).  Zero rows and an all-negative-zero row are included."""
    rows = []
    allbits = np.arange(0x0001, 0x7F80, dtype=np.uint32)
    allvals = (allbits << 16).view(np.float32)
    amaxes = [448.0, 449.0, 1.0, 3.0, 7.0, 0.1, 1e-3, 2.0 ** -120, 123.456, 5.0e4, 3.3e38, 1.7e-38]
    for a in amaxes:
        a = float(torch.tensor(a).to(torch.bfloat16).float())
        vals = allvals[allvals <= a]
        vals = np.concatenate([vals, -vals])
        n = (len(vals) + 126) // 127
        vals = np.resize(vals, n * 127).reshape(n, 127)
        rows.append(np.concatenate([np.full((n, 1), a, np.float32), vals], axis=1))
    rows.append(np.zeros((1, 128), np.float32))
    rows.append(np.full((1, 128), -0.0, np.float32))
    x = np.concatenate(rows, axis=0)
    return torch.from_numpy(x).to(torch.bfloat16)


@pytest.mark.parametrize("fmt", FMTS, ids=["e4m3", "e5m2"])
@pytest.mark.parametrize("sf", SFS, ids=["fp32", "ue8m0"])
def test_act_quant_rounding_boundaries(cuda_device, fmt, sf):
    x = _boundary_rows()
    q, s = run_act(x, fmt[0], sf[0], cuda_device)
    qr, sr = O.act_quant(x, fmt=fmt[1], scale_fmt=sf[1])
    assert_scales_equal(s, sr, "scales")
    assert_codes_equal(q, qr, "codes")


@pytest.mark.parametrize("sf", SFS, ids=["fp32", "ue8m0"])
def test_act_quant_sweep_sizes(cuda_device, sf):
    """Quantiser-sweep shapes, Student-t(3) entries: full comparison at M = 1024 and
    4096, every 61st row at M = 16384 (the oracle checks those rows one by one)."""
    K = 7168
    for M in (1024, 4096):
        x = synth.activations(M, K, seed=0, dist="t3", device=cuda_device)
        q, s = F.act_quant(x, scale_fmt=sf[0])
        qr, sr = O.act_quant(x.cpu(), scale_fmt=sf[1], threads=THREADS)
        assert_codes_equal(codes(q), qr, f"codes M={M}")
        assert_scales_equal(s.cpu().numpy(), sr, f"scales M={M}")
    x = synth.activations(16384, K, seed=0, dist="t3", device=cuda_device)
    q, s = F.act_quant(x, scale_fmt=sf[0])
    rows = torch.arange(0, 16384, 61)
    xr = x[rows.to(cuda_device)].cpu()
    qr, sr = O.act_quant(xr, scale_fmt=sf[1])
    assert_codes_equal(codes(q[rows.to(cuda_device)]), qr, "codes M=16384 (sampled rows)")
    assert_scales_equal(s[rows.to(cuda_device)].cpu().numpy(), sr, "scales M=16384 (sampled rows)")


@pytest.mark.parametrize("fmt", FMTS, ids=["e4m3", "e5m2"])
@pytest.mark.parametrize("sf", SFS, ids=["fp32", "ue8m0"])
@pytest.mark.parametrize("shape", [(256, 512), (300, 272), (18432 // 8, 7168)])
def test_weight_block_quant(cuda_device, fmt, sf, shape):
    """128 x 128 blocks, E4M3 and E5M2 codes, fp32 and ue8m0 scales; ragged edge blocks;
    one block carries an outlier.  Every code and scale."""
    N, K = shape
    w = synth.weights(N, K, 0.02, seed=1, device=cuda_device)
    w[min(N - 1, 130), min(K - 1, 260)] = 3.0      # one block with an outlier
    q, s = F.weight_quant(w, block=128, fmt=fmt[0], scale_fmt=sf[0])
    qr, sr = O.weight_quant(w.cpu(), block=128, fmt=fmt[1], scale_fmt=sf[1], threads=THREADS)
    assert_codes_equal(codes(q), qr, "codes")
    assert_scales_equal(s.cpu().numpy(), sr, "scales")


@pytest.mark.parametrize("fmt", FMTS, ids=["e4m3", "e5m2"])
@pytest.mark.parametrize("sf", SFS, ids=["fp32", "ue8m0"])
@pytest.mark.parametrize("shape", [(64, 256), (1024, 7168), (16384, 7168)])
def test_per_tensor_quant(cuda_device, fmt, sf, shape):
    M, K = shape
    x = synth.activations(M, K, seed=2, dist="t3", device=cuda_device)
    q, s = F.weight_quant(x, block=0, fmt=fmt[0], scale_fmt=sf[0])
    torch.cuda.synchronize()
    if M * K <= 8_000_000:
        qr, sr = O.tensor_quant(x.cpu(), fmt=fmt[1], scale_fmt=sf[1])
        assert_codes_equal(codes(q), qr, "codes")
    else:
        # the scale depends on every element: take the amax on the host (exact), then
        # check the oracle's cast under that scale on a row sample
        amax = float(x.abs().max().float())
        sr = np.array([O.scale_from_amax(amax, fmt[1], sf[1])], np.float32)
        rows = torch.arange(0, M, 97, device=cuda_device)
        qr = O.cast_with_scale(x[rows].cpu(), float(sr[0]), fmt[1])
        assert_codes_equal(codes(q[rows]), qr, "codes (sampled rows)")
    assert_scales_equal(s.cpu().numpy(), sr, "scale")
