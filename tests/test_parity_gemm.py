"""GPU parity of the block-scaled FP8 GEMMs against the fp64 CPU oracle.

The GPU path quantises the seeded bf16 inputs with its own kernels; the codes and
scales are first checked bit-exact against the oracle's quantisers, then the GEMM
output is compared element by element with the oracle's fp64 GEMM over the same
codes:  fp32 output within 1e-5 * sum_k |a_k w_k|, bf16 output within one bf16
ulp of the oracle rounded straight to bf16 (cancellation allowance: _parity.py).
Full-size cases compare the rows the oracle can compute one by one.
"""
import numpy as np
import pytest
import torch

import fp8_block_scaled_12_b200 as F
import oracle as O
import synth
from _parity import THREADS, assert_codes_equal, assert_scales_equal, bits_u16, check_bf16, check_fp32, codes

pytestmark = pytest.mark.gpu


def quantise_both(x, w, sf, dev):
    """GPU act/weight quantisation, checked bit-exact against the oracle's; returns
    device (qa, sa, qw, sw) and host numpy copies."""
    osf = O.SCALE_FP32 if sf == F.SCALE_FP32 else O.SCALE_UE8M0
    xd, wd = x.to(dev), w.to(dev)
    qa, sa = F.act_quant(xd, scale_fmt=sf)
    qw, sw = F.weight_quant(wd, scale_fmt=sf)
    torch.cuda.synchronize()
    h = dict(qa=codes(qa), sa=sa.cpu().numpy(), qw=codes(qw), sw=sw.cpu().numpy())
    return (qa, sa, qw, sw), h


def oracle_check_quant(x, w, sf, h, rows=None):
    osf = O.SCALE_FP32 if sf == F.SCALE_FP32 else O.SCALE_UE8M0
    xs = x if rows is None else x[rows]
    qar, sar = O.act_quant(xs, scale_fmt=osf, threads=THREADS)
    assert_codes_equal(h["qa"] if rows is None else h["qa"][rows], qar, "activation codes")
    assert_scales_equal(h["sa"] if rows is None else h["sa"][rows], sar, "activation scales")
    qwr, swr = O.weight_quant(w, scale_fmt=osf, threads=THREADS)
    assert_codes_equal(h["qw"], qwr, "weight codes")
    assert_scales_equal(h["sw"], swr, "weight scales")


def gemm_and_compare(dev, M, N, K, sf=F.SCALE_FP32, rows=None, outs=("bf16", "fp32"), seed=0,
                     outliers=None, factor=1.0, w_std=0.02, check_weights=True):
    x = synth.activations(M, K, seed=seed, outliers=outliers, factor=factor)
    w = synth.weights(N, K, w_std, seed=seed)
    (qa, sa, qw, sw), h = quantise_both(x, w, sf, dev)
    if check_weights:
        oracle_check_quant(x, w, sf, h, rows)
    y_ref, bound = O.gemm_rows(h["qa"], h["sa"], h["qw"], h["sw"], rows=rows, threads=THREADS)
    sel = slice(None) if rows is None else torch.as_tensor(rows, device=dev)
    allowed = 0
    for o in outs:
        y = F.block_gemm(qa, sa, qw, sw, out_dtype=torch.bfloat16 if o == "bf16" else torch.float32)
        torch.cuda.synchronize()
        assert F.fp8_device_error() == 0
        yh = y[sel]
        if o == "fp32":
            check_fp32(yh.cpu().numpy(), y_ref, bound, f"fp32 M={M} N={N} K={K}")
        else:
            allowed += check_bf16(bits_u16(yh), y_ref, bound, f"bf16 M={M} N={N} K={K}")
    return allowed


def test_tiny_config(cuda_device):
    p = synth.TINY.params
    gemm_and_compare(cuda_device, p["M"], p["N"], p["K"], outliers=p["outliers"], factor=p["factor"])


@pytest.mark.parametrize("M", [1, 8, 16, 40, 64, 65, 100, 128, 150, 160, 161, 200, 256])
def test_swap_path_token_counts(cuda_device, M):
    """M <= 160 runs the weight-stationary kernel, larger M the 128x256 tile kernel; ragged token counts, N and K span
    several tiles."""
    gemm_and_compare(cuda_device, M, 384, 1024, seed=M)


@pytest.mark.parametrize("shape", [(1, 256, 8192), (64, 256, 8192), (40, 272, 7296), (100, 384, 3840), (160, 256, 3712)])
def test_swap_path_scale_segments(cuda_device, shape):
    """The weight-stationary kernel stages scales in segments of 56 (<= 64 tokens) or
    28 (<= 160 tokens) K-blocks: K spans several segments with a ragged last one."""
    M, N, K = shape
    gemm_and_compare(cuda_device, M, N, K, seed=11 + M)


@pytest.mark.parametrize("M", [8, 300])
def test_single_k_block(cuda_device, M):
    """K = 128: one K-block, one scale per row on either path."""
    gemm_and_compare(cuda_device, M, 256, 128, seed=M)


@pytest.mark.parametrize("shape", [(257, 512, 512), (300, 272, 640), (512, 1024, 1024), (1000, 528, 384)])
def test_wide_path_ragged(cuda_device, shape):
    M, N, K = shape
    gemm_and_compare(cuda_device, M, N, K, seed=7)


def test_ue8m0_scales(cuda_device):
    gemm_and_compare(cuda_device, 300, 512, 1024, sf=F.SCALE_UE8M0, seed=5, outliers=[3, 77, 500], factor=30.0)


def test_integer_exact(cuda_device):
    """Small-integer codes with unit scales: every product and partial sum is an exact
    fp32 integer, so the fp32 output must equal numpy's int64 matmul exactly."""
    rng = np.random.default_rng(9)
    M, N, K = 200, 256, 2048
    A = rng.integers(-8, 9, (M, K)).astype(np.float32)
    W = rng.integers(-8, 9, (N, K)).astype(np.float32)
    dev = cuda_device
    qa = torch.from_numpy(A).to(torch.float8_e4m3fn).view(torch.uint8).to(dev)
    qw = torch.from_numpy(W).to(torch.float8_e4m3fn).view(torch.uint8).to(dev)
    sa = torch.ones((M, K // 128), dtype=torch.float32, device=dev)
    sw = torch.ones((N // 128, K // 128), dtype=torch.float32, device=dev)
    ref = (A.astype(np.int64) @ W.astype(np.int64).T).astype(np.float64)
    for m in (M, 1000):
        if m != M:   # wide path too
            A2 = rng.integers(-8, 9, (m, K)).astype(np.float32)
            qa = torch.from_numpy(A2).to(torch.float8_e4m3fn).view(torch.uint8).to(dev)
            sa = torch.ones((m, K // 128), dtype=torch.float32, device=dev)
            ref = (A2.astype(np.int64) @ W.astype(np.int64).T).astype(np.float64)
        y = F.block_gemm(qa, sa, qw, sw, out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert (y.cpu().numpy().astype(np.float64) == ref).all()


@pytest.mark.parametrize("M", [1, 8, 32, 64])
def test_decode_config_full_size(cuda_device, M):
    """Decode-shaped linear at full size (N=18432, K=7168, ue8m0), rows sampled."""
    p = synth.DECODE.params
    K, N = p["K"], p["N"]
    ch = synth.outlier_channels(K, synth.n_outliers(K, p["outlier_frac"]), seed=0)
    rows = sorted({0, M // 2, M - 1})
    gemm_and_compare(cuda_device, M, N, K, sf=F.SCALE_UE8M0, rows=rows, outs=("bf16",), seed=0,
                     outliers=ch, factor=p["factor"], w_std=p["w_std"], check_weights=(M == 1))


def test_prefill_config_full_size(cuda_device):
    """Prefill-shaped linear at full size (4096 x 28672 x 8192, fp32 scales), on the
    launch the benchmark times; 3 sampled rows against the oracle."""
    p = synth.PREFILL.params
    M, N, K = p["M"], p["N"], p["K"]
    dev = cuda_device
    ch = synth.outlier_channels(K, synth.n_outliers(K, p["outlier_frac"]), seed=0)
    x = synth.activations(M, K, seed=0, outliers=ch, factor=p["factor"], device=dev)
    w = synth.weights(N, K, p["w_std"], seed=0, device=dev)
    qa, sa = F.act_quant(x)
    qw, sw = F.weight_quant(w)
    y = F.block_gemm(qa, sa, qw, sw)
    torch.cuda.synchronize()
    assert F.fp8_device_error() == 0
    rows = [0, 1777, 4095]
    hq = dict(qa=codes(qa[rows]), sa=sa[rows].cpu().numpy(), qw=codes(qw), sw=sw.cpu().numpy())
    qar, sar = O.act_quant(x[rows].cpu())
    assert_codes_equal(hq["qa"], qar, "activation codes")
    assert_scales_equal(hq["sa"], sar, "activation scales")
    # every weight code and block scale against the oracle (row blocks split over host threads)
    qwr, swr = O.weight_quant(w.cpu(), threads=THREADS)
    assert_codes_equal(hq["qw"], qwr, "weight codes (all 28672 rows)")
    assert_scales_equal(hq["sw"], swr, "weight scales (all 224 x 64 blocks)")
    del qwr
    y_ref, bound = O.gemm_rows(hq["qa"], hq["sa"], hq["qw"], hq["sw"], threads=THREADS)
    check_bf16(bits_u16(y[rows]), y_ref, bound, "prefill bf16")


# --------------------------------------------------------------------------
# Persistent loops: sizes at which every CTA of the (SM-count sized) grid runs
# at least three work items, compared element by element.


def test_wide_persistent_multi_tile(cuda_device):
    """M=2048, N=7168: 16 x 28 = 448 tiles of 128 x 256 over at most 148 CTAs (>= 3 tiles
    each).  K = 384 is three K-blocks, an odd count, so the tensor-memory buffer and its
    phase alternate differently from one tile to the next.  Every element, fp32 and bf16."""
    gemm_and_compare(cuda_device, 2048, 7168, 384, seed=21)


@pytest.mark.parametrize("M", [40, 150])
def test_swap_dense_multi_unit(cuda_device, M):
    """Few-token path with N = 57344: 448 units of 128 weight rows over at most 148 CTAs
    (>= 3 units each), for both token tiles (M <= 64 and 64 < M <= 160).  Every element."""
    gemm_and_compare(cuda_device, M, 57344, 384, seed=M + 3)


def test_swap_dense_multi_unit_multi_segment(cuda_device):
    """M = 65 (token tile 160, 28 K-blocks per scale segment) and K = 29 K-blocks: each
    of the >= 3 units per CTA has a full and a one-K-block segment, so the two
    scale-table buffers alternate inside and across units.  Every element."""
    gemm_and_compare(cuda_device, 65, 56832, 29 * 128, seed=29, outs=("bf16",))
