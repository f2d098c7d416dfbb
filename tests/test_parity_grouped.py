"""GPU parity of the grouped (MoE expert) GEMM against the fp64 CPU oracle."""
import numpy as np
import pytest
import torch

import fp8_block_scaled_12_b200 as F
import oracle as O
import synth
from _parity import THREADS, assert_codes_equal, assert_scales_equal, bits_u16, check_bf16, check_fp32, codes

pytestmark = pytest.mark.gpu


def make_grouped(dev, counts, N, K, seed=0, w_std=0.02):
    E = len(counts)
    off = np.zeros(E + 1, np.int32)
    off[1:] = np.cumsum(counts)
    T = int(off[-1])
    x = synth.activations(max(T, 1), K, seed=seed, dist="normal")[:T]
    w = torch.stack([synth.weights(N, K, w_std, seed=seed, chunk=e) for e in range(E)])
    qa, sa = F.act_quant(x.to(dev))
    qw = torch.empty((E, N, K), dtype=torch.uint8, device=dev)
    sw = torch.empty((E, (N + 127) // 128, K // 128), dtype=torch.float32, device=dev)
    for e in range(E):
        F.fp8_weight_quant(w[e].to(dev), qw[e], sw[e])
    torch.cuda.synchronize()
    return x, w, off, (qa, sa, qw, sw)


@pytest.mark.parametrize("counts", [[0, 37, 300, 1, 129], [256, 0, 0, 16], [5, 600, 17, 255, 257, 0, 3]])
def test_grouped_ragged_groups(cuda_device, counts):
    dev = cuda_device
    N, K = 256, 512
    x, w, off, (qa, sa, qw, sw) = make_grouped(dev, counts, N, K, seed=len(counts))
    qar, sar = O.act_quant(x)
    assert_codes_equal(codes(qa), qar, "activation codes")
    assert_scales_equal(sa.cpu().numpy(), sar, "activation scales")
    offd = torch.from_numpy(off).to(dev)
    T = int(off[-1])
    rows = np.arange(T)
    y_ref, bound = O.grouped_gemm_rows(codes(qa), sa.cpu().numpy(), codes(qw), sw.cpu().numpy(), off, rows,
                                       threads=THREADS)
    for out in (torch.float32, torch.bfloat16):
        y = torch.full((T, N), float("nan"), dtype=out, device=dev)
        F.fp8_grouped_gemm(qa, sa, qw, sw, offd, y)
        torch.cuda.synchronize()
        assert F.fp8_device_error() == 0
        if out == torch.float32:
            check_fp32(y.cpu().numpy(), y_ref, bound, "grouped fp32")
        else:
            check_bf16(bits_u16(y), y_ref, bound, "grouped bf16")


def test_grouped_ragged_n_and_scale_segments(cuda_device):
    """N = 272 (the last 128-row weight block of every expert is partial) and K spans
    two scale segments of 28 K-blocks plus a ragged one; the last expert's tail block
    reads past the weight tensor (zero fill) and must not disturb the others."""
    dev = cuda_device
    counts = [3, 170, 0, 64, 161]
    N, K = 272, 128 * 60
    x, w, off, (qa, sa, qw, sw) = make_grouped(dev, counts, N, K, seed=9)
    offd = torch.from_numpy(off).to(dev)
    T = int(off[-1])
    rows = np.arange(0, T, 3)
    y_ref, bound = O.grouped_gemm_rows(codes(qa), sa.cpu().numpy(), codes(qw), sw.cpu().numpy(), off, rows,
                                       threads=THREADS)
    for out in (torch.float32, torch.bfloat16):
        y = torch.full((T, N), float("nan"), dtype=out, device=dev)
        F.fp8_grouped_gemm(qa, sa, qw, sw, offd, y)
        torch.cuda.synchronize()
        assert F.fp8_device_error() == 0
        if out == torch.float32:
            check_fp32(y[rows].cpu().numpy(), y_ref, bound, "grouped fp32 ragged N")
        else:
            check_bf16(bits_u16(y[rows]), y_ref, bound, "grouped bf16 ragged N")


def test_grouped_leaves_rows_outside_groups_untouched(cuda_device):
    dev = cuda_device
    counts = [10, 20]
    N, K = 128, 256
    x, w, off, (qa, sa, qw, sw) = make_grouped(dev, counts, N, K, seed=1)
    # two extra rows beyond offsets[E]
    qa2 = torch.cat([qa, qa[:2]])
    sa2 = torch.cat([sa, sa[:2]])
    y = torch.full((32, N), 7.0, dtype=torch.float32, device=dev)
    F.fp8_grouped_gemm(qa2, sa2, qw, sw, torch.from_numpy(off).to(dev), y)
    torch.cuda.synchronize()
    assert (y[30:] == 7.0).all()


def test_grouped_equals_dense_for_one_group(cuda_device):
    dev = cuda_device
    x, w, off, (qa, sa, qw, sw) = make_grouped(dev, [300], 384, 1024, seed=2)
    yg = F.grouped_gemm(qa, sa, qw, sw, torch.from_numpy(off).to(dev), out_dtype=torch.float32)
    yd = F.block_gemm(qa, sa, qw[0], sw[0], out_dtype=torch.float32)
    torch.cuda.synchronize()
    y_ref, bound = O.gemm_rows(codes(qa), sa.cpu().numpy(), codes(qw[0]), sw[0].cpu().numpy())
    check_fp32(yg.cpu().numpy(), y_ref, bound, "grouped")
    check_fp32(yd.cpu().numpy(), y_ref, bound, "dense")


def test_moe_config_full_size(cuda_device):
    """MoE config at full size: 4096 tokens, top-8 of 256 experts, N=2048, K=7168.
    The first and last row of 12 experts are compared with the oracle."""
    p = synth.MOE.params
    T, E, k, N, K = p["T"], p["E"], p["topk"], p["N"], p["K"]
    dev = cuda_device
    row_token, row_expert, off = synth.routing(T, E, k, seed=0)
    xt = synth.activations(T, K, seed=0, device=dev)
    xs = xt[row_token.to(dev)]
    qa, sa = F.act_quant(xs)
    qw = torch.empty((E, N, K), dtype=torch.uint8, device=dev)
    sw = torch.empty((E, N // 128, K // 128), dtype=torch.float32, device=dev)
    experts = [0, 1, 17, 64, 100, 128, 150, 200, 201, 230, 254, 255]
    checked = experts[::2]                       # weight codes of 6 experts (88 M codes)
    w_keep = {}
    for e in range(E):
        we = synth.weights(N, K, p["w_std"], seed=0, chunk=e, device=dev)
        F.fp8_weight_quant(we, qw[e], sw[e])
        if e in checked:
            w_keep[e] = we.cpu()
    offd = off.to(dev)
    y = F.grouped_gemm(qa, sa, qw, sw, offd)
    torch.cuda.synchronize()
    assert F.fp8_device_error() == 0
    for e in checked:
        qwr, swr = O.weight_quant(w_keep[e], threads=THREADS)
        assert_codes_equal(codes(qw[e]), qwr, f"expert {e} weight codes")
        assert_scales_equal(sw[e].cpu().numpy(), swr, f"expert {e} weight scales")
    offn = off.numpy()
    for e in experts:
        r0, r1 = int(offn[e]), int(offn[e + 1])
        if r1 <= r0:
            continue
        rows = sorted({r0, r1 - 1})
        qar, sar = O.act_quant(xs[rows].cpu())
        assert_codes_equal(codes(qa[rows]), qar, "activation codes")
        y_ref, bound = O.gemm_rows(codes(qa[rows]), sa[rows].cpu().numpy(), codes(qw[e]), sw[e].cpu().numpy())
        check_bf16(bits_u16(y[rows]), y_ref, bound, f"moe expert {e}")


def _grouped_full_compare(dev, counts, N, K, seed, outs=(torch.float32, torch.bfloat16)):
    x, w, off, (qa, sa, qw, sw) = make_grouped(dev, counts, N, K, seed=seed)
    qar, sar = O.act_quant(x, threads=THREADS)
    assert_codes_equal(codes(qa), qar, "activation codes")
    assert_scales_equal(sa.cpu().numpy(), sar, "activation scales")
    offd = torch.from_numpy(off).to(dev)
    T = int(off[-1])
    rows = np.arange(T)
    y_ref, bound = O.grouped_gemm_rows(codes(qa), sa.cpu().numpy(), codes(qw), sw.cpu().numpy(), off, rows,
                                       threads=THREADS)
    for out in outs:
        y = torch.full((T, N), float("nan"), dtype=out, device=dev)
        F.fp8_grouped_gemm(qa, sa, qw, sw, offd, y)
        torch.cuda.synchronize()
        assert F.fp8_device_error() == 0
        if out == torch.float32:
            check_fp32(y.cpu().numpy(), y_ref, bound, f"grouped fp32 E={len(counts)} N={N} K={K}")
        else:
            check_bf16(bits_u16(y), y_ref, bound, f"grouped bf16 E={len(counts)} N={N} K={K}")


def _ragged_counts(E, seed, hi=90):
    """Seeded ragged expert sizes with empty experts, single-row experts and experts
    larger than one 160-token chunk."""
    rng = np.random.default_rng(seed)
    c = rng.integers(0, hi, E)
    c[rng.choice(E, E // 8, replace=False)] = 0
    c[rng.choice(E, 3, replace=False)] = 1
    c[rng.choice(E, 2, replace=False)] = 170
    return c.tolist()


def test_grouped_persistent_multi_unit(cuda_device):
    """E = 64 experts x N = 1024 (8 weight blocks each): 512 units over at most 148 CTAs
    (>= 3 each), ragged and empty experts.  Every element, fp32 and bf16."""
    _grouped_full_compare(cuda_device, _ragged_counts(64, 5), 1024, 512, seed=31)


def test_grouped_persistent_multi_unit_multi_segment(cuda_device):
    """Same unit count with K = 29 K-blocks: each unit has a 28-K-block and a 1-K-block
    scale segment, so the scale tables alternate inside units, across units and across
    experts.  Every element."""
    _grouped_full_compare(cuda_device, _ragged_counts(64, 6, hi=30), 1024, 29 * 128, seed=32,
                          outs=(torch.bfloat16,))
