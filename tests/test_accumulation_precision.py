"""Accumulation precision of the tensor-core partial sums (one 128-deep K-block).

The pages fix FP8 products with fp32 accumulation ("LLM 推理的 FP8 混合精度工程 2026",
section 3).  Each K-block's partial sum comes from the tensor core; these crafted
rows make any accumulation narrower than fp32 visible: one large product (448) next
to 127 products of the smallest E4M3 subnormal (2^-9), in several orders, and an
exact cancellation (448 - 448) next to small terms.  Every exact sum here is an fp32
number, so a correctly rounded fp32 accumulation reproduces it exactly; the test
requires the pages' tolerance (1e-5 * sum |a w|) and reports the worst error.
"""
import numpy as np
import pytest
import torch

import fp8_block_scaled_12_b200 as F

pytestmark = pytest.mark.gpu

E4M3_448, E4M3_MIN_SUB, E4M3_ONE = 0x7E, 0x01, 0x38
NEG = 0x80


def crafted_rows(K=128):
    rows = []
    r = np.full(K, E4M3_MIN_SUB, np.uint8); r[0] = E4M3_448; rows.append(r)                     # big first
    r = np.full(K, E4M3_MIN_SUB, np.uint8); r[-1] = E4M3_448; rows.append(r)                    # big last
    r = np.full(K, E4M3_MIN_SUB, np.uint8); r[64] = E4M3_448; rows.append(r)                    # big in the middle
    r = np.full(K, E4M3_MIN_SUB, np.uint8); r[0] = E4M3_448; r[1] = E4M3_448 | NEG; rows.append(r)   # cancel
    r = np.full(K, E4M3_MIN_SUB, np.uint8); r[5] = E4M3_448; r[100] = E4M3_448 | NEG; rows.append(r)
    r = np.full(K, E4M3_MIN_SUB | NEG, np.uint8); r[31] = E4M3_448; rows.append(r)               # big minus small
    return np.stack(rows)


@pytest.mark.parametrize("M", [6, 300])
def test_small_terms_survive_a_large_one(cuda_device, M):
    """M = 6 runs the weight-stationary kernel, M = 300 the 128x256 tile kernel."""
    base = crafted_rows()
    qa_h = np.concatenate([base] * ((M + len(base) - 1) // len(base)))[:M]
    K, N = 128, 256
    qw_h = np.full((N, K), E4M3_ONE, np.uint8)
    dev = cuda_device
    qa = torch.from_numpy(qa_h).to(dev)
    qw = torch.from_numpy(qw_h).to(dev)
    sa = torch.ones((M, 1), dtype=torch.float32, device=dev)
    sw = torch.ones((N // 128, 1), dtype=torch.float32, device=dev)
    y = F.block_gemm(qa, sa, qw, sw, out_dtype=torch.float32)
    assert F.fp8_device_error() == 0
    a = qa_h.view(np.uint8).astype(np.int64)
    mag = np.where((a & 0x7F) == E4M3_448, 448.0, 2.0 ** -9)
    val = np.where(a & NEG, -mag, mag)
    exact = val.sum(axis=1)                       # every partial sum is exact in fp64
    bound = np.abs(val).sum(axis=1)
    got = y.cpu().numpy().astype(np.float64)
    err = np.abs(got - exact[:, None])
    assert (err <= 1e-5 * bound[:, None]).all(), f"worst error {err.max()} vs tolerance {1e-5 * bound.max()}"
