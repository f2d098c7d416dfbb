"""GPU parity of the two steps beside the GEMM: the BF16 path's weight dequantisation,
and the next layer's act_quant fused into the GEMM epilogue.

weight_dequant: every bf16 output bit-exact with the oracle.
Fused epilogue: the bf16 output y is checked against the fp64 oracle GEMM as for
fp8_block_gemm (1 bf16 ulp), and the fused codes and scales must be bit-exact with the
oracle's act_quant applied to that same bf16 y -- the output the kernel rounds and
quantises; without y the codes must be identical to the run with y."""
import numpy as np
import pytest
import torch

import fp8_block_scaled_12_b200 as F
import oracle as O
import synth
from _parity import THREADS, assert_codes_equal, assert_scales_equal, bits_u16, check_bf16, codes

pytestmark = pytest.mark.gpu

FMTS = [(F.E4M3, O.E4M3), (F.E5M2, O.E5M2)]
SFS = [(F.SCALE_FP32, O.SCALE_FP32), (F.SCALE_UE8M0, O.SCALE_UE8M0)]


@pytest.mark.parametrize("fmt", FMTS, ids=["e4m3", "e5m2"])
@pytest.mark.parametrize("sf", SFS, ids=["fp32", "ue8m0"])
@pytest.mark.parametrize("shape", [(256, 512), (300, 272), (2304, 7168)])
def test_weight_dequant(cuda_device, fmt, sf, shape):
    N, K = shape
    w = synth.weights(N, K, 0.02, seed=6, device=cuda_device)
    w[min(N - 1, 140), min(K - 1, 300)] = 5.0
    q, s = F.weight_quant(w, fmt=fmt[0], scale_fmt=sf[0])
    out = F.weight_dequant(q, s, fmt=fmt[0])
    torch.cuda.synchronize()
    ref = O.weight_dequant(codes(q), s.cpu().numpy(), fmt=fmt[1], threads=THREADS)
    got = bits_u16(out)
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"{len(bad)} bf16 mismatches, first at {bad[:3].tolist()}"


def test_weight_dequant_per_tensor(cuda_device):
    x = synth.activations(1000, 1040, seed=7, dist="t3", device=cuda_device)
    q, s = F.weight_quant(x, block=0)
    out = F.weight_dequant(q, s, block=0)
    torch.cuda.synchronize()
    ref = O.weight_dequant(codes(q), s.cpu().numpy(), block=0)
    assert np.array_equal(bits_u16(out), ref)


def fused_compare(dev, M, N, K, fmt, sf, seed):
    x = synth.activations(M, K, seed=seed, outliers=[3, K // 3], factor=25.0)
    w = synth.weights(N, K, 0.02, seed=seed)
    qa, sa = F.act_quant(x.to(dev))
    qw, sw = F.weight_quant(w.to(dev))
    qy, sy, y = F.block_gemm_quant(qa, sa, qw, sw, fmt=fmt[0], scale_fmt=sf[0], with_y=True)
    qy2, sy2 = F.block_gemm_quant(qa, sa, qw, sw, fmt=fmt[0], scale_fmt=sf[0])
    torch.cuda.synchronize()
    assert F.fp8_device_error() == 0
    y_ref, bound = O.gemm_rows(codes(qa), sa.cpu().numpy(), codes(qw), sw.cpu().numpy(), threads=THREADS)
    check_bf16(bits_u16(y), y_ref, bound, f"fused y M={M} N={N} K={K}")
    qr, sr = O.act_quant(y.cpu(), fmt=fmt[1], scale_fmt=sf[1], threads=THREADS)
    assert_codes_equal(codes(qy), qr, f"fused codes M={M}")
    assert_scales_equal(sy.cpu().numpy(), sr, f"fused scales M={M}")
    assert np.array_equal(codes(qy2), codes(qy)) and np.array_equal(sy2.cpu().numpy().view(np.uint32),
                                                                     sy.cpu().numpy().view(np.uint32))


@pytest.mark.parametrize("fmt", FMTS, ids=["e4m3", "e5m2"])
@pytest.mark.parametrize("sf", SFS, ids=["fp32", "ue8m0"])
@pytest.mark.parametrize("M", [1, 40, 64, 100, 160, 300])
def test_fused_act_quant_epilogue(cuda_device, fmt, sf, M):
    """Every epilogue: M <= 64 and <= 160 (weight-stationary, a group spread over a
    warpgroup) and M > 160 (128 x 256 tiles, a group inside one thread)."""
    fused_compare(cuda_device, M, 384, 1024, fmt, sf, seed=M + 50)


def test_fused_act_quant_multi_tile(cuda_device):
    """448 tiles of the wide kernel and 448 weight units of the swap kernel over at
    most 148 CTAs: every CTA quantises several groups."""
    fused_compare(cuda_device, 2048, 7168, 384, FMTS[0], SFS[0], seed=61)
    fused_compare(cuda_device, 40, 57344, 384, FMTS[0], SFS[1], seed=62)
