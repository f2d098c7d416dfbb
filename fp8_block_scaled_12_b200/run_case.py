"""Run one operation of the library on seeded synthetic data and time it.

    python -m fp8_block_scaled_12_b200.run_case --op gemm --M 4096 --N 28672 --K 8192 --iters 3
    python -m fp8_block_scaled_12_b200.run_case --op act_quant --M 16384 --K 7168 --scale ue8m0
    python -m fp8_block_scaled_12_b200.run_case --op weight_quant --M 28672 --K 8192 --block 0 --fmt e5m2
    python -m fp8_block_scaled_12_b200.run_case --op grouped --tokens 4096 --E 256 --N 2048 --K 7168
    python -m fp8_block_scaled_12_b200.run_case --op mx_gemm --M 4096 --N 28672 --K 8192 --scale ue8m0
    python -m fp8_block_scaled_12_b200.run_case --op mx_quant --M 16384 --K 7168

Inputs are prepared before the measured launches (so a profiler can skip them by
launch count: the op's own launches come last, `--iters` of them, after `--warm`
untimed ones).  Prints one line of CUDA-event timing per op.
"""
from __future__ import annotations

import argparse
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import fp8_block_scaled_12_b200 as F  # noqa: E402
import synth  # noqa: E402


def timed(fn, warm, iters):
    for _ in range(warm):
        fn()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record()
    for _ in range(iters):
        fn()
    b.record()
    torch.cuda.synchronize()
    if F.fp8_device_error() != 0:
        raise RuntimeError("device wait timed out")
    return a.elapsed_time(b) / max(iters, 1)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--op", required=True, choices=["act_quant", "weight_quant", "gemm", "grouped", "mx_quant",
                                                    "mx_gemm", "delayed", "gemm_quant", "dequant", "moe"])
    ap.add_argument("--M", type=int, default=4096)
    ap.add_argument("--N", type=int, default=28672)
    ap.add_argument("--K", type=int, default=8192)
    ap.add_argument("--E", type=int, default=256)
    ap.add_argument("--tokens", type=int, default=4096)
    ap.add_argument("--topk", type=int, default=8)
    ap.add_argument("--block", type=int, default=128)
    ap.add_argument("--fmt", choices=["e4m3", "e5m2"], default="e4m3")
    ap.add_argument("--scale", choices=["fp32", "ue8m0"], default="fp32")
    ap.add_argument("--out", choices=["bf16", "fp32"], default="bf16")
    ap.add_argument("--dist", choices=["normal", "t3"], default="normal")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--warm", type=int, default=1)
    a = ap.parse_args()
    dev = torch.device("cuda:0")
    fmt = F.E4M3 if a.fmt == "e4m3" else F.E5M2
    sf = F.SCALE_FP32 if a.scale == "fp32" else F.SCALE_UE8M0
    odt = torch.bfloat16 if a.out == "bf16" else torch.float32

    if a.op == "act_quant":
        x = synth.activations(a.M, a.K, seed=0, dist=a.dist, device=dev)
        q = torch.empty((a.M, a.K), dtype=torch.uint8, device=dev)
        s = torch.empty((a.M, (a.K + 127) // 128), dtype=torch.float32, device=dev)
        ms = timed(lambda: F.fp8_act_quant(x, q, s, fmt=fmt, scale_fmt=sf), a.warm, a.iters)
        b = a.M * a.K * 3 + s.numel() * 4
        print(f"act_quant M={a.M} K={a.K} {a.fmt}/{a.scale}: {ms * 1e3:.2f} us  {b / ms / 1e6:.1f} GB/s")
    elif a.op == "weight_quant":
        w = synth.weights(a.M, a.K, 0.02, seed=0, device=dev) if a.dist == "normal" else \
            synth.activations(a.M, a.K, seed=0, dist="t3", device=dev)
        q = torch.empty((a.M, a.K), dtype=torch.uint8, device=dev)
        shape = (1,) if a.block == 0 else ((a.M + 127) // 128, (a.K + 127) // 128)
        s = torch.empty(shape, dtype=torch.float32, device=dev)
        ms = timed(lambda: F.fp8_weight_quant(w, q, s, block=a.block, fmt=fmt, scale_fmt=sf), a.warm, a.iters)
        b = a.M * a.K * 3 + s.numel() * 4
        print(f"weight_quant N={a.M} K={a.K} block={a.block} {a.fmt}/{a.scale}: {ms * 1e3:.2f} us  "
              f"{b / ms / 1e6:.1f} GB/s (3 B/elt)")
    elif a.op == "gemm":
        x = synth.activations(a.M, a.K, seed=0, device=dev)
        w = synth.weights(a.N, a.K, 0.02, seed=0, device=dev)
        qa, sa = F.act_quant(x, scale_fmt=sf)
        qw, sw = F.weight_quant(w, scale_fmt=sf)
        del x, w
        y = torch.empty((a.M, a.N), dtype=odt, device=dev)
        ms = timed(lambda: F.fp8_block_gemm(qa, sa, qw, sw, y), a.warm, a.iters)
        fl = 2.0 * a.M * a.N * a.K
        b = qa.numel() + qw.numel() + y.numel() * y.element_size() + sa.numel() * 4 + sw.numel() * 4
        print(f"gemm M={a.M} N={a.N} K={a.K} {a.scale} {a.out}: {ms * 1e3:.2f} us  {fl / ms / 1e9:.1f} TFLOPS  "
              f"{b / ms / 1e6:.1f} GB/s")
    elif a.op == "moe":
        # routed layer: scores -> route, act_quant into sorted rows, GEMM + weighted scatter
        g = torch.Generator(device=dev).manual_seed(3)
        scores = torch.rand((a.tokens, a.E), generator=g, device=dev, dtype=torch.float32)
        x = synth.activations(a.tokens, a.K, seed=0, device=dev)
        qa, sa = F.act_quant(x)
        qw = torch.empty((a.E, a.N, a.K), dtype=torch.uint8, device=dev)
        sw = torch.empty((a.E, (a.N + 127) // 128, a.K // 128), dtype=torch.float32, device=dev)
        for e in range(a.E):
            F.fp8_weight_quant(synth.weights(a.N, a.K, 0.02, seed=0, chunk=e, device=dev), qw[e], sw[e])
        route = F.moe_route(scores, a.topk)
        qs, ss = F.act_quant_permute(x, route)
        out = torch.empty((a.tokens, a.N), dtype=torch.float32, device=dev)
        ms = timed(lambda: F.fp8_moe_gemm(qs, ss, qw, sw, route, out), a.warm, a.iters)
        fl = 2.0 * a.tokens * a.topk * a.N * a.K
        print(f"moe_gemm tokens={a.tokens} E={a.E} top-{a.topk} N={a.N} K={a.K}: {ms * 1e3:.1f} us  "
              f"{fl / ms / 1e9:.1f} TFLOPS")
    elif a.op == "gemm_quant":
        x = synth.activations(a.M, a.K, seed=0, device=dev)
        w = synth.weights(a.N, a.K, 0.02, seed=0, device=dev)
        qa, sa = F.act_quant(x, scale_fmt=sf)
        qw, sw = F.weight_quant(w, scale_fmt=sf)
        del x, w
        qy = torch.empty((a.M, a.N), dtype=torch.uint8, device=dev)
        sy = torch.empty((a.M, a.N // 128), dtype=torch.float32, device=dev)
        ms = timed(lambda: F.fp8_block_gemm_quant(qa, sa, qw, sw, qy, sy, None, fmt, sf), a.warm, a.iters)
        fl = 2.0 * a.M * a.N * a.K
        print(f"gemm_quant M={a.M} N={a.N} K={a.K} {a.scale}: {ms * 1e3:.2f} us  {fl / ms / 1e9:.1f} TFLOPS")
    elif a.op == "dequant":
        w = synth.weights(a.M, a.K, 0.02, seed=0, device=dev)
        q, s = F.weight_quant(w, block=a.block, fmt=fmt, scale_fmt=sf)
        out = torch.empty_like(w)
        ms = timed(lambda: F.fp8_weight_dequant(q, s, out, a.block, fmt), a.warm, a.iters)
        b = a.M * a.K * 3 + s.numel() * 4
        print(f"dequant N={a.M} K={a.K} block={a.block} {a.fmt}: {ms * 1e3:.2f} us  {b / ms / 1e6:.1f} GB/s")
    elif a.op == "delayed":
        x = synth.activations(a.M, a.K, seed=0, dist=a.dist, device=dev)
        q = torch.empty((a.M, a.K), dtype=torch.uint8, device=dev)
        ds = F.DelayedScaling(hist_len=16, fmt=fmt, device=dev)
        nclip = torch.empty(1, dtype=torch.int64, device=dev)
        sused = torch.empty(1, dtype=torch.float32, device=dev)
        ms = timed(lambda: F.fp8_delayed_quant(x, q, ds.scale, ds.pos, ds.history, nclip, sused, fmt=fmt,
                                               target=ds.target), a.warm, a.iters)
        b = a.M * a.K * 3
        print(f"delayed M={a.M} K={a.K} {a.fmt}: {ms * 1e3:.2f} us  {b / ms / 1e6:.1f} GB/s (3 B/elt)")
    elif a.op == "mx_quant":
        x = synth.activations(a.M, a.K, seed=0, dist=a.dist, device=dev)
        q = torch.empty((a.M, a.K), dtype=torch.uint8, device=dev)
        e8 = torch.empty((F.mx_sf_bytes(a.M, a.K),), dtype=torch.uint8, device=dev)
        ms = timed(lambda: F.fp8_mx_quant(x, q, e8, fmt=fmt), a.warm, a.iters)
        b = a.M * a.K * 3 + a.M * ((a.K + 31) // 32)
        print(f"mx_quant M={a.M} K={a.K} {a.fmt}: {ms * 1e3:.2f} us  {b / ms / 1e6:.1f} GB/s")
    elif a.op == "mx_gemm":
        # --scale fp32 selects MXFP8 (32-element E8M0 exponents), ue8m0 the power-of-two
        # scales of the block GEMM's layout
        x = synth.activations(a.M, a.K, seed=0, device=dev)
        w = synth.weights(a.N, a.K, 0.02, seed=0, device=dev)
        if a.scale == "fp32":
            qa, sa = F.mx_quant(x)
            qw, sw = F.mx_quant(w)
        else:
            qa, s_a = F.act_quant(x, scale_fmt=F.SCALE_UE8M0)
            qw, s_w = F.weight_quant(w, scale_fmt=F.SCALE_UE8M0)
            sa = F.mx_pack_pow2(s_a, a.M, a.K, 1)
            sw = F.mx_pack_pow2(s_w, a.N, a.K, 128)
        del x, w
        y = torch.empty((a.M, a.N), dtype=odt, device=dev)
        ms = timed(lambda: F.fp8_mx_gemm(qa, sa, qw, sw, y), a.warm, a.iters)
        fl = 2.0 * a.M * a.N * a.K
        layout = "e8m0x32" if a.scale == "fp32" else "pow2x128"
        print(f"mx_gemm M={a.M} N={a.N} K={a.K} {layout} {a.out}: {ms * 1e3:.2f} us  {fl / ms / 1e9:.1f} TFLOPS")
    else:
        row_token, _, off = synth.routing(a.tokens, a.E, a.topk, seed=0)
        xt = synth.activations(a.tokens, a.K, seed=0, device=dev)
        qa, sa = F.act_quant(xt[row_token.to(dev)], scale_fmt=sf)
        del xt
        qw = torch.empty((a.E, a.N, a.K), dtype=torch.uint8, device=dev)
        sw = torch.empty((a.E, (a.N + 127) // 128, a.K // 128), dtype=torch.float32, device=dev)
        for e in range(a.E):
            F.fp8_weight_quant(synth.weights(a.N, a.K, 0.02, seed=0, chunk=e, device=dev), qw[e], sw[e],
                               scale_fmt=sf)
        y = torch.empty((qa.shape[0], a.N), dtype=odt, device=dev)
        offd = off.to(dev)
        ms = timed(lambda: F.fp8_grouped_gemm(qa, sa, qw, sw, offd, y), a.warm, a.iters)
        fl = 2.0 * qa.shape[0] * a.N * a.K
        b = qw.numel() + qa.numel() + y.numel() * y.element_size() + sa.numel() * 4 + sw.numel() * 4
        print(f"grouped rows={qa.shape[0]} E={a.E} N={a.N} K={a.K}: {ms * 1e3:.1f} us  {fl / ms / 1e9:.1f} TFLOPS  "
              f"{b / ms / 1e6:.1f} GB/s")


if __name__ == "__main__":
    main()
