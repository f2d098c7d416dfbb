"""GPU parity of the MXFP8 path (32-element E8M0 blocks) and of the power-of-two
(ue8m0) block GEMM on the tensor core's scale path, against the CPU oracle.

Codes and exponent bytes must be bit-exact (the library stores the exponents in the
tensor core's tiled order; untile_e8m0 permutes them back to the oracle's [rows,
K/32] before comparing).  GEMM tolerance, derived from the
arithmetic (no tolerance is stated for this variant): every E4M3 x E4M3 product and
its power-of-two scale are exact in fp32, and the fp32 accumulator in tensor memory
takes one rounding per 32-element block product it adds (K/32 of them), plus at most
32 more inside a block if the hardware rounds there too, so
    |y - y_ref| <= (K/32 + 32) * 2^-24 * sum_k |a_k w_k|
(fp32 output); bf16 output must be within one bf16 ulp of the oracle rounded straight
to bf16, with the same cancellation allowance as the other GEMM tests at that bound.
"""
import numpy as np
import pytest
import torch

import fp8_block_scaled_12_b200 as F
import oracle as O
import synth
from _parity import (THREADS, assert_codes_equal, bits_u16, check_bf16, check_fp32, codes, tile_e8m0,
                     untile_e8m0)

pytestmark = pytest.mark.gpu


def mx_rel(K: int) -> float:
    return (K / 32 + 32) * 2.0 ** -24


def bytes_(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy()


def assert_bytes_equal(got, ref, what):
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"{what}: {len(bad)} mismatching exponent bytes, first at {bad[:5].tolist()}"


# ----------------------------------------------------------------- quantiser
@pytest.mark.parametrize("fmt", [(F.E4M3, O.E4M3), (F.E5M2, O.E5M2)], ids=["e4m3", "e5m2"])
@pytest.mark.parametrize("shape", [(16, 512), (37, 208), (5, 48), (129, 4112), (1000, 7168)])
def test_mx_quant_shapes(cuda_device, fmt, shape):
    """Every code and exponent byte; ragged K (a last block of 16 elements, K % 128 != 0)."""
    M, K = shape
    x = synth.activations(M, K, seed=7, dist="t3", outliers=[1, K // 2], factor=40.0)
    q, e8 = F.mx_quant(x.to(cuda_device), fmt=fmt[0])
    torch.cuda.synchronize()
    qr, er = O.mx_quant(x, fmt=fmt[1], threads=THREADS)
    assert_codes_equal(codes(q), qr, f"codes {shape}")
    assert_bytes_equal(untile_e8m0(e8, M, K), er, f"exponents {shape}")


@pytest.mark.parametrize("fmt", [(F.E4M3, O.E4M3), (F.E5M2, O.E5M2)], ids=["e4m3", "e5m2"])
def test_mx_quant_rounding_boundaries(cuda_device, fmt):
    """Blocks of 32 holding one amax and 31 values swept over every bf16 magnitude up to
    it (ties, subnormal codes, signed zeros, values that round up to Fmax), plus zero
    blocks: each block's exponent and every code."""
    rows = []
    allbits = np.arange(0x0001, 0x7F80, dtype=np.uint32)
    allvals = (allbits << 16).view(np.float32)
    for a in [448.0, 450.0, 1.0, 3.0, 0.1, 2.0 ** -120, 5.0e4, 6.0e4, 3.3e38]:
        a = float(torch.tensor(a).to(torch.bfloat16).float())
        vals = allvals[allvals <= a]
        vals = np.concatenate([vals, -vals])
        n = (len(vals) + 30) // 31
        vals = np.resize(vals, n * 31).reshape(n, 31)
        rows.append(np.concatenate([np.full((n, 1), a, np.float32), vals], axis=1))
    blocks = np.concatenate(rows + [np.zeros((1, 32), np.float32), np.full((1, 32), -0.0, np.float32)], axis=0)
    nb = blocks.shape[0] - blocks.shape[0] % 4
    x = torch.from_numpy(blocks[:nb].reshape(-1, 128)).to(torch.bfloat16)
    q, e8 = F.mx_quant(x.to(cuda_device), fmt=fmt[0])
    torch.cuda.synchronize()
    qr, er = O.mx_quant(x, fmt=fmt[1], threads=THREADS)
    assert_bytes_equal(untile_e8m0(e8, x.shape[0], 128), er, "exponents")
    assert_codes_equal(codes(q), qr, "codes")


def test_mx_quant_row_stride_and_sweep_size(cuda_device):
    """A strided input, then the sweep tensor 16384 x 7168 (every 61st row checked)."""
    x = synth.activations(33, 384, seed=4, outliers=[1, 200], factor=30.0)
    buf = torch.zeros((33, 392), dtype=torch.bfloat16, device=cuda_device)
    buf[:, :384] = x.to(cuda_device)
    q, e8 = F.mx_quant(buf[:, :384])
    qr, er = O.mx_quant(x)
    assert_codes_equal(codes(q), qr, "codes (strided)")
    assert_bytes_equal(untile_e8m0(e8, 33, 384), er, "exponents (strided)")
    xs = synth.activations(16384, 7168, seed=0, dist="t3", device=cuda_device)
    q, e8 = F.mx_quant(xs)
    rows = torch.arange(0, 16384, 61, device=cuda_device)
    qr, er = O.mx_quant(xs[rows].cpu(), threads=THREADS)
    assert_codes_equal(codes(q[rows]), qr, "codes 16384x7168 (sampled rows)")
    assert_bytes_equal(untile_e8m0(e8, 16384, 7168)[rows.cpu().numpy()], er, "exponents 16384x7168 (sampled rows)")


# ---------------------------------------------------------------- MXFP8 GEMM
def mx_gemm_compare(dev, M, N, K, seed, outs=("bf16", "fp32"), rows=None, outliers=None, factor=1.0, w_std=0.02):
    x = synth.activations(M, K, seed=seed, outliers=outliers, factor=factor)
    w = synth.weights(N, K, w_std, seed=seed)
    qa, ea = F.mx_quant(x.to(dev))
    qw, ew = F.mx_quant(w.to(dev))
    torch.cuda.synchronize()
    h = dict(qa=codes(qa), ea=untile_e8m0(ea, M, K), qw=codes(qw), ew=untile_e8m0(ew, N, K))
    if rows is None:
        qar, ear = O.mx_quant(x, threads=THREADS)
        assert_codes_equal(h["qa"], qar, "activation codes")
        assert_bytes_equal(h["ea"], ear, "activation exponents")
    y_ref, bound = O.mx_gemm_rows(h["qa"], h["ea"], h["qw"], h["ew"], rows=rows, threads=THREADS)
    sel = slice(None) if rows is None else torch.as_tensor(rows, device=dev)
    for o in outs:
        y = F.mx_gemm(qa, ea, qw, ew, out_dtype=torch.bfloat16 if o == "bf16" else torch.float32)
        torch.cuda.synchronize()
        assert F.fp8_device_error() == 0
        yh = y[sel]
        if o == "fp32":
            check_fp32(yh.cpu().numpy(), y_ref, bound, f"mx fp32 M={M} N={N} K={K}", rel=mx_rel(K))
        else:
            check_bf16(bits_u16(yh), y_ref, bound, f"mx bf16 M={M} N={N} K={K}", rel=mx_rel(K))
    return h


def test_mx_gemm_tiny(cuda_device):
    p = synth.TINY.params
    mx_gemm_compare(cuda_device, p["M"], p["N"], p["K"], seed=0, outliers=p["outliers"], factor=p["factor"])


@pytest.mark.parametrize("M", [1, 8, 40, 64, 65, 100, 160, 161, 300])
def test_mx_gemm_token_counts(cuda_device, M):
    """M <= 64 and 64 < M <= 160 run the weight-stationary orientation, larger M the
    128 x 256 tile; ragged counts, several tiles in N and K."""
    mx_gemm_compare(cuda_device, M, 384, 1024, seed=M)


@pytest.mark.parametrize("M", [1, 40, 100, 300])
def test_mx_gemm_single_k_block(cuda_device, M):
    """K = 128: the weight-stationary shapes' second MMA issuer gets no K-block, so the
    epilogue must use the first accumulator alone."""
    mx_gemm_compare(cuda_device, M, 384, 128, seed=M + 7)


@pytest.mark.parametrize("shape", [(257, 512, 512), (300, 272, 640), (1000, 528, 384), (40, 272, 7296)])
def test_mx_gemm_ragged(cuda_device, shape):
    M, N, K = shape
    mx_gemm_compare(cuda_device, M, N, K, seed=9, outliers=[3, 100], factor=30.0)


def test_mx_gemm_integer_exact(cuda_device):
    """Small-integer codes with exponent bytes 127 (scale 1): every product and partial
    sum is an exact fp32 integer, so the output equals numpy's int64 matmul exactly;
    then random per-block exponents against exact rational block sums."""
    rng = np.random.default_rng(11)
    dev = cuda_device
    for M in (40, 300):
        N, K = 256, 1024
        A = rng.integers(-8, 9, (M, K))
        W = rng.integers(-8, 9, (N, K))
        qa = torch.from_numpy(A.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).to(dev)
        qw = torch.from_numpy(W.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).to(dev)
        ea = torch.from_numpy(tile_e8m0(np.full((M, K // 32), 127, np.uint8), M, K)).to(dev)
        ew = torch.from_numpy(tile_e8m0(np.full((N, K // 32), 127, np.uint8), N, K)).to(dev)
        y = F.mx_gemm(qa, ea, qw, ew, out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert (y.cpu().numpy().astype(np.float64) == (A @ W.T).astype(np.float64)).all()
        # per-block exponents 2^-3 .. 2^3 on both sides: block sums stay exact in fp32
        eab = rng.integers(124, 131, (M, K // 32)).astype(np.uint8)
        ewb = rng.integers(124, 131, (N, K // 32)).astype(np.uint8)
        y = F.mx_gemm(qa, torch.from_numpy(tile_e8m0(eab, M, K)).to(dev), qw,
                      torch.from_numpy(tile_e8m0(ewb, N, K)).to(dev), out_dtype=torch.float32)
        torch.cuda.synchronize()
        ref = np.zeros((M, N))
        for g in range(K // 32):
            blk = A[:, 32 * g:32 * g + 32] @ W[:, 32 * g:32 * g + 32].T
            ref += blk * np.exp2(eab[:, g:g + 1].astype(np.float64) - 127) * np.exp2(ewb[:, g].astype(np.float64) - 127)
        assert (y.cpu().numpy().astype(np.float64) == ref).all()


def test_mx_gemm_persistent_multi_tile(cuda_device):
    """448 wide tiles over at most 148 CTAs (>= 3 each), odd K-block count, every element."""
    mx_gemm_compare(cuda_device, 2048, 7168, 384, seed=21)


def test_mx_gemm_swap_multi_unit(cuda_device):
    """448 weight units over at most 148 CTAs, 40 tokens, every element."""
    mx_gemm_compare(cuda_device, 40, 57344, 384, seed=22)


# ----------------------------------------------- ue8m0 block GEMM on the scale path
def pow2_compare(dev, M, N, K, seed, rows=None, outs=("bf16", "fp32"), outliers=None, factor=1.0, w_std=0.02,
                 device_inputs=False):
    x = synth.activations(M, K, seed=seed, outliers=outliers, factor=factor, device=dev if device_inputs else "cpu")
    w = synth.weights(N, K, w_std, seed=seed, device=dev if device_inputs else "cpu")
    qa, sa = F.act_quant(x.to(dev), scale_fmt=F.SCALE_UE8M0)
    qw, sw = F.weight_quant(w.to(dev), scale_fmt=F.SCALE_UE8M0)
    ea = F.mx_pack_pow2(sa, M, K, 1)
    ew = F.mx_pack_pow2(sw, N, K, 128)
    torch.cuda.synchronize()
    assert F.fp8_device_error() == 0
    hqa = codes(qa) if rows is None else codes(qa[torch.as_tensor(rows, device=dev)])
    hsa = sa.cpu().numpy() if rows is None else sa[torch.as_tensor(rows, device=dev)].cpu().numpy()
    y_ref, bound = O.gemm_rows(hqa, hsa, codes(qw), sw.cpu().numpy(), threads=THREADS)
    sel = slice(None) if rows is None else torch.as_tensor(rows, device=dev)
    for o in outs:
        y = F.mx_gemm(qa, ea, qw, ew, out_dtype=torch.bfloat16 if o == "bf16" else torch.float32)
        torch.cuda.synchronize()
        assert F.fp8_device_error() == 0
        if o == "fp32":
            check_fp32(y[sel].cpu().numpy(), y_ref, bound, f"pow2 fp32 M={M} N={N} K={K}", rel=mx_rel(K))
        else:
            check_bf16(bits_u16(y[sel]), y_ref, bound, f"pow2 bf16 M={M} N={N} K={K}", rel=mx_rel(K))


def test_pack_pow2_layout(cuda_device):
    """The packed bytes are each scale's exponent field, replicated over the four
    32-element blocks of its K-block and (row_block 128) over the block's rows."""
    dev = cuda_device
    M, N, K = 200, 300, 640
    rng = np.random.default_rng(5)
    sa = np.exp2(rng.integers(-20, 20, (M, K // 128))).astype(np.float32)
    sw = np.exp2(rng.integers(-20, 20, ((N + 127) // 128, K // 128))).astype(np.float32)
    ea = F.mx_pack_pow2(torch.from_numpy(sa).to(dev), M, K, 1)
    ew = F.mx_pack_pow2(torch.from_numpy(sw).to(dev), N, K, 128)
    torch.cuda.synchronize()
    assert F.fp8_device_error() == 0
    exp_a = np.repeat((sa.view(np.uint32) >> 23).astype(np.uint8), 4, axis=1)
    exp_w = np.repeat(np.repeat((sw.view(np.uint32) >> 23).astype(np.uint8), 4, axis=1), 128, axis=0)[:N]
    assert_bytes_equal(untile_e8m0(ea, M, K), exp_a, "packed activation exponents")
    assert_bytes_equal(untile_e8m0(ew, N, K), exp_w, "packed weight exponents")


@pytest.mark.parametrize("M", [1, 64, 150, 300])
def test_pow2_block_gemm_on_scale_path(cuda_device, M):
    """act_quant / weight_quant with ue8m0 scales, packed and multiplied on the scale
    path: the oracle is the block GEMM's own definition (orc_gemm_rows)."""
    pow2_compare(cuda_device, M, 384, 1024, seed=M + 1, outliers=[5, 700], factor=30.0)


@pytest.mark.parametrize("M", [1, 64])
def test_pow2_decode_config_full_size(cuda_device, M):
    """Decode-shaped linear (18432 x 7168, ue8m0, 36 outlier channels x30) on the scale
    path, rows sampled."""
    p = synth.DECODE.params
    K, N = p["K"], p["N"]
    ch = synth.outlier_channels(K, synth.n_outliers(K, p["outlier_frac"]), seed=0)
    rows = sorted({0, M // 2, M - 1})
    pow2_compare(cuda_device, M, N, K, seed=0, rows=rows, outs=("bf16",), outliers=ch, factor=p["factor"],
                 w_std=p["w_std"], device_inputs=True)


def test_pack_rejects_scales_that_are_not_powers_of_two(cuda_device):
    """fp32 scales that are not powers of two are flagged through fp8_device_error
    instead of being silently truncated to their exponent."""
    dev = cuda_device
    x = synth.activations(64, 512, seed=1, device=dev)
    qa, sa = F.act_quant(x)                     # fp32 scales: amax / 448, not powers of two
    F.mx_pack_pow2(sa, 64, 512, 1)
    assert F.fp8_device_error() == F.FP8_ERR_INVALID_SCALE
    assert F.fp8_device_error() == 0            # reading clears it
