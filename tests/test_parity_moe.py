"""GPU parity of MoE routing (bit-exact: expert ids, gate weights, offsets and the
sorted permutation), of act_quant written straight into the expert-sorted rows
(bit-exact with the oracle's act_quant of the tokens, permuted), and of the grouped
GEMM with the gate-weighted scatter-add of its outputs fused in, against the oracle.

Combine tolerance, derived: each expert output carries the block GEMM's error
(1e-5 * sum|a w| per element, the tolerance the other GEMM tests use); the gate product
and the k fp32 additions into the output (in any order) add at most (k + 1) * 2^-24 of
sum_j |w_j y_j| <= sum_j |w_j| sum|a w|.  So |out - ref| <= (1e-5 + (k+1) 2^-24) * bound
with bound = sum_j |w_j| * sum_k |a_k w_k| from the oracle."""
import numpy as np
import pytest
import torch

import fp8_block_scaled_12_b200 as F
import oracle as O
import synth
from _parity import THREADS, check_fp32, codes

pytestmark = pytest.mark.gpu


def route_both(dev, scores, k):
    r = F.moe_route(scores.to(dev), k)
    torch.cuda.synchronize()
    ro = O.moe_route(scores.numpy(), k)
    for name in ("ids", "offsets", "row_token", "token_row"):
        got = r[name].cpu().numpy()
        assert np.array_equal(got, ro[name]), f"{name}: {np.argwhere(got != ro[name])[:5].tolist()}"
    for name in ("w", "row_weight"):
        got = r[name].cpu().numpy().view(np.uint32)
        assert np.array_equal(got, ro[name].view(np.uint32)), f"{name} bits differ"
    return r, ro


def scores_for(T, E, seed, ties=False):
    g = torch.Generator().manual_seed(seed)
    s = torch.rand((T, E), generator=g, dtype=torch.float32)
    if ties:
        s = (s * 8).floor() / 8                         # heavy ties
        s[0, :] = 0.0                                    # all-zero row: 1/k weights
    return s


@pytest.mark.parametrize("T,E,k", [(1, 4, 2), (300, 64, 8), (4096, 256, 8), (77, 1000, 5), (513, 33, 32)])
def test_routing(cuda_device, T, E, k):
    route_both(cuda_device, scores_for(T, E, seed=T + E), k)


def test_routing_ties(cuda_device):
    route_both(cuda_device, scores_for(1000, 256, seed=1, ties=True), 8)


def test_routing_many_chunks(cuda_device):
    """131072 pairs: 256 chunks of the sort, each placing its rows after all earlier
    chunks' rows of the same expert."""
    route_both(cuda_device, scores_for(16384, 256, seed=5), 8)


def test_routing_no_tokens(cuda_device):
    r = F.moe_route(torch.empty((0, 64), dtype=torch.float32, device=cuda_device), 4)
    torch.cuda.synchronize()
    assert F.fp8_device_error() == 0
    assert r["offsets"].cpu().tolist() == [0] * 65


def moe_compare(dev, T, E, k, N, K, seed, tokens=None, scores=None):
    scores = scores_for(T, E, seed) if scores is None else scores
    r, ro = route_both(dev, scores, k)
    x = synth.activations(T, K, seed=seed, device=dev)
    qa, sa = F.act_quant(x)                      # token-major, for the oracle's combine
    qs, ss = F.act_quant_permute(x, r)           # expert-sorted, for the GEMM
    torch.cuda.synchronize()
    qar, sar = O.act_quant(x.cpu(), threads=THREADS)
    perm = np.empty(T * k, np.int64)
    perm[ro["token_row"]] = np.repeat(np.arange(T), k)   # sorted row -> token
    assert np.array_equal(codes(qs), qar[perm]), "permuted activation codes"
    assert np.array_equal(ss.cpu().numpy().view(np.uint32), sar[perm].view(np.uint32)), "permuted scales"
    qw = torch.empty((E, N, K), dtype=torch.uint8, device=dev)
    sw = torch.empty((E, (N + 127) // 128, K // 128), dtype=torch.float32, device=dev)
    for e in range(E):
        F.fp8_weight_quant(synth.weights(N, K, 0.02, seed=seed, chunk=e, device=dev), qw[e], sw[e])
    out = F.moe_gemm(qs, ss, qw, sw, r)
    torch.cuda.synchronize()
    assert F.fp8_device_error() == 0
    toks = np.arange(T) if tokens is None else np.asarray(tokens)
    ref, bound = O.moe_combine_rows(qar, sar, codes(qw), sw.cpu().numpy(), ro["ids"], ro["w"], toks,
                                    threads=THREADS)
    rel = 1e-5 + (k + 1) * 2.0 ** -24
    check_fp32(out.cpu().numpy()[toks], ref, bound, f"moe T={T} E={E} k={k} N={N} K={K}", rel=rel)


@pytest.mark.parametrize("T,E,k,N,K", [(40, 8, 2, 256, 512), (300, 16, 4, 272, 1024), (1000, 64, 8, 1024, 384)])
def test_moe_layer_permute_scatter(cuda_device, T, E, k, N, K):
    """Ragged experts (some empty), ragged N, chunks of 160 routed rows; the last case
    has 512 units over at most 148 CTAs.  Every token."""
    moe_compare(cuda_device, T, E, k, N, K, seed=T)


def test_moe_config_full_size(cuda_device):
    """4096 tokens, top-8 of 256 experts, N = 2048, K = 7168: 48 sampled tokens."""
    p = synth.MOE.params
    toks = np.linspace(0, p["T"] - 1, 48).astype(np.int64)
    moe_compare(cuda_device, p["T"], p["E"], p["topk"], p["N"], p["K"], seed=0, tokens=toks)


def test_moe_skewed_experts(cuda_device):
    """Expert 0 preferred by most tokens: its 560+ rows span four chunks of 160 in the
    scatter GEMM, while other experts get a few rows or none."""
    T, E, k = 700, 16, 2
    s = scores_for(T, E, seed=13)
    s[:600, 0] += 2.0                                   # expert 0 wins for 600 tokens
    moe_compare(cuda_device, T, E, k, 256, 512, seed=13, scores=s)


@pytest.mark.parametrize("T,E,k", [(200, 8, 1), (50, 4, 4)])
def test_moe_top1_and_all_experts(cuda_device, T, E, k):
    """k = 1 (each token one expert, weight 1) and k = E (every expert every token)."""
    moe_compare(cuda_device, T, E, k, 256, 512, seed=T + k)
