"""Seeded synthetic inputs for the FP8 W8A8 linear-layer workloads.

This module only draws random bf16 tensors and routing tables; it holds none of
the method's arithmetic (no amax, no scale, no FP8 cast, no GEMM).  Both the CUDA
path and the CPU oracle consume the exact bf16 bytes it returns: tests generate
once, hand the tensor to the library on the GPU and a host copy to the oracle.

Workload shapes follow the pages' LLM settings ("FP8 推理提速 83.6%: DeepSeek-V3 在
AMD MI250 上的完整落地指南", 官方配置中最关键的四个参数: 256 routed experts, 8
active per token; hidden size 7168) and the activation outliers the FP8
engineering page describes ("LLM 推理的 FP8 混合精度工程 2026", section 4: spikes
of 30-100x on particular channels).

Determinism: every draw uses a torch.Generator seeded from (seed, stream,
chunk).  On the CPU that is torch's CPU generator; on a CUDA device it is
torch's device (Philox) generator, so large tensors (MoE expert weights: 3.76 G
elements) are drawn in milliseconds.  The two devices give different but each
fully reproducible values.  Sub-streams: 0 activations, 1 weights, 2 outlier
channel choice, 3 routing.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

STREAM_ACT, STREAM_W, STREAM_OUTLIER, STREAM_ROUTE = 0, 1, 2, 3


def _gen(device, seed: int, stream: int, chunk: int = 0) -> torch.Generator:
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(_mix(seed, stream, chunk))
    return g


def _mix(seed: int, stream: int, chunk: int) -> int:
    """A distinct, fixed generator seed per (seed, stream, chunk): the SplitMix64
    finaliser of a packed key (torch's CPU generator keeps only the low 32 bits, so
    every bit of the key must reach them)."""
    M64 = (1 << 64) - 1
    z = ((seed & 0xFFFFFFFF) << 32 | (stream & 0xFF) << 24 | (chunk & 0xFFFFFF)) & M64
    z = (z + 0x9E3779B97F4A7C15) & M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
    z ^= z >> 31
    return z & 0x7FFFFFFFFFFFFFFF


def normal_f32(shape, std: float, seed: int, stream: int, chunk: int = 0, device="cpu") -> torch.Tensor:
    g = _gen(device, seed, stream, chunk)
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x


def student_t3_f32(shape, seed: int, stream: int, chunk: int = 0, device="cpu") -> torch.Tensor:
    """Student-t with 3 degrees of freedom: Z / sqrt(chi2_3 / 3), chi2_3 a sum of 3 squared normals."""
    g = _gen(device, seed, stream, chunk)
    z = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    c = torch.zeros_like(z)
    for _ in range(3):
        c.add_(torch.randn(*shape, generator=g, device=device, dtype=torch.float32).square_())
    return z.div_(c.div_(3.0).sqrt_())


def outlier_channels(K: int, count: int, seed: int) -> torch.Tensor:
    """`count` distinct channel indices out of K, drawn by a seeded permutation (host)."""
    g = _gen("cpu", seed, STREAM_OUTLIER)
    return torch.randperm(K, generator=g)[:count].sort().values


def activations(M: int, K: int, seed: int = 0, outliers=None, factor: float = 1.0,
                dist: str = "normal", device="cpu") -> torch.Tensor:
    """bf16 [M, K]: N(0,1) (or Student-t(3)) with the listed channels multiplied by `factor`
    in fp32 before the single round-to-nearest-even to bf16."""
    if dist == "normal":
        x = normal_f32((M, K), 1.0, seed, STREAM_ACT, device=device)
    elif dist == "t3":
        x = student_t3_f32((M, K), seed, STREAM_ACT, device=device)
    else:
        raise ValueError(dist)
    if outliers is not None and len(outliers) > 0:
        idx = torch.as_tensor(outliers, dtype=torch.long, device=x.device)
        x[:, idx] *= factor
    return x.to(torch.bfloat16)


def weights(N: int, K: int, std: float, seed: int = 0, chunk: int = 0, device="cpu") -> torch.Tensor:
    """bf16 [N, K] ~ N(0, std^2) (std is a standard deviation)."""
    return normal_f32((N, K), std, seed, STREAM_W, chunk, device=device).to(torch.bfloat16)


def routing(T: int, E: int, topk: int, seed: int = 0):
    """Uniform top-k routing without repeats, then a stable sort of the (token, expert)
    pairs by expert.  Returns (row_token int64 [T*topk], row_expert int64 [T*topk],
    offsets int32 [E+1]) on the host: row r of the sorted matrix is token row_token[r]."""
    g = _gen("cpu", seed, STREAM_ROUTE)
    keys = torch.rand(T, E, generator=g)
    experts = keys.topk(topk, dim=1).indices                      # [T, topk], distinct per token
    tok = torch.arange(T).unsqueeze(1).expand(T, topk).reshape(-1)
    exp = experts.reshape(-1)
    order = torch.argsort(exp * T + tok, stable=True)
    row_token, row_expert = tok[order], exp[order]
    counts = torch.bincount(row_expert, minlength=E)
    offsets = torch.zeros(E + 1, dtype=torch.int32)
    offsets[1:] = torch.cumsum(counts, 0).to(torch.int32)
    return row_token, row_expert, offsets


# ----------------------------------------------------------------- workloads
@dataclass
class Workload:
    name: str
    desc: str
    params: dict = field(default_factory=dict)


TINY = Workload("tiny", "tiny W8A8 linear: x bf16 16x512 N(0,1), channels 7 and 300 x20; "
                "W bf16 256x512 N(0,0.02); fp32 scales; fp32 and bf16 output",
                dict(M=16, N=256, K=512, outliers=[7, 300], factor=20.0, w_std=0.02))
DECODE = Workload("decode", "decode-shaped linear: x bf16 M in {1,8,32,64} x 7168 N(0,1), 0.5% of "
                  "channels x30; W bf16 18432x7168 N(0,0.015); ue8m0 scales; bf16 output",
                  dict(Ms=[1, 8, 32, 64], N=18432, K=7168, outlier_frac=0.005, factor=30.0, w_std=0.015))
PREFILL = Workload("prefill", "prefill-shaped linear: x bf16 4096x8192 N(0,1), 1% of channels x20; "
                   "W bf16 28672x8192 N(0,0.02); fp32 scales; bf16 output",
                   dict(M=4096, N=28672, K=8192, outlier_frac=0.01, factor=20.0, w_std=0.02))
MOE = Workload("moe", "grouped MoE expert GEMM: 4096 tokens x 7168 N(0,1), uniform top-8 of 256 "
               "experts, rows sorted by expert; per-expert W 2048x7168 N(0,0.02); bf16 output",
               dict(T=4096, E=256, topk=8, N=2048, K=7168, w_std=0.02))
SWEEP = Workload("sweep", "quantiser sweep: bf16 M in {1024,4096,16384} x 7168 Student-t(3); "
                 "per-128 e4m3 fp32 and ue8m0; per-tensor e4m3 and e5m2",
                 dict(Ms=[1024, 4096, 16384], K=7168))
WORKLOADS = {w.name: w for w in (TINY, DECODE, PREFILL, MOE, SWEEP)}


def n_outliers(K: int, frac: float) -> int:
    return int(round(frac * K))
