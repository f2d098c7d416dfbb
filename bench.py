"""Benchmark of the FP8 W8A8 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill|decode|moe|sweep]
                    [--impl ours|reference] [--no-rows]

Default workload (the headline): the prefill-shaped linear, x bf16 4096 x 8192
(1% outlier channels x20), W 28672 x 8192 as E4M3 with 128x128 fp32 block scales
(quantised once, as the pages ship FP8 checkpoints).  One step = act_quant(x)
(per token, per 128 channels, fp32 scales) + block-scaled FP8 GEMM, bf16 out.
Metric: GEMM TFLOPS over the step (2*M*N*K per step); act_quant GB/s is reported
beside it.  Inputs are larger than L2 (W alone is 235 MB), so no flush is needed.

Under torchrun every rank runs its own token batch through the same layer (data
parallel, no collective on the data path: weak scaling); the barrier and the
max-over-ranks timing use torch.distributed.

--impl reference times the CPU oracle (plain C, fp64 GEMM) on a bounded sample
of the same workload on the host cores; only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import hashlib
import itertools
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "block-scaled FP8 GEMM TFLOPS (% dense FP8 peak); act_quant GB/s (% HBM peak)"
FP8_OVER_BF16 = 2.0          # nominal dense FP8 / BF16 tensor throughput ratio on B200 (4.5 / 2.25 PF)
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}


# --------------------------------------------------------------------- helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK), "fallback"


def source_sha() -> str:
    h = hashlib.sha256()
    for f in ("gemm.cuh", "gemm_swap.cuh", "ptx.cuh", "quant.cuh", "fp8lin.cu"):
        h.update(open(os.path.join(ROOT, "fp8_block_scaled_12_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_key: str):
    """Per-launch DRAM bytes of `kernel_key` from the committed ncu summary, if the
    summary was taken on the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.md")
    if not os.path.exists(p):
        return None
    sha = source_sha()
    for line in open(p):
        m = re.match(r"\|\s*" + re.escape(kernel_key) + r"\s*\|\s*([0-9.eE+]+)\s*\|\s*([0-9a-f]+)\s*\|", line)
        if m and m.group(2) == sha:
            return float(m.group(1))
    return None


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML in a background thread."""
    REASONS = {
        0x0000000000000004: "sw_power_cap", 0x0000000000000008: "hw_slowdown",
        0x0000000000000020: "sw_thermal_slowdown", 0x0000000000000040: "hw_thermal_slowdown",
        0x0000000000000080: "hw_power_brake_slowdown", 0x0000000000000002: "applications_clocks_setting",
    }

    def __init__(self, index: int, period_s: float = 0.01):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self._stop = period_s, threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = self._handle(pynvml, index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    @staticmethod
    def _handle(nv, index: int):
        """NVML handle of the CUDA device `index`: NVML numbers every GPU of the host,
        CUDA only the visible ones, so the device is matched by UUID (PCI bus id as a
        fallback) rather than by index."""
        import torch
        props = torch.cuda.get_device_properties(index)
        try:
            return nv.nvmlDeviceGetHandleByUUID("GPU-" + str(props.uuid))
        except Exception:
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


def reduce_max(vals, dev=None):
    """Element-wise max over all ranks of a list of floats (identity without a process
    group).  Timings are reported as the slowest rank's."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in vals]
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def weak_scaling_tflops(flops_per_rank_step: float, world: int, steps: int, ms: float) -> float:
    """Whole-job throughput: every rank runs `steps` steps of its own batch in `ms`."""
    return flops_per_rank_step * world * steps / (ms * 1e-3) / 1e12


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ------------------------------------------------------------------ workloads
def setup_prefill(dev, rank):
    import torch
    import fp8_block_scaled_12_b200 as F
    import synth
    p = synth.PREFILL.params
    M, N, K = p["M"], p["N"], p["K"]
    ch = synth.outlier_channels(K, synth.n_outliers(K, p["outlier_frac"]), seed=0)
    x = synth.activations(M, K, seed=rank, outliers=ch, factor=p["factor"], device=dev)
    w = synth.weights(N, K, p["w_std"], seed=0, device=dev)
    qw, sw = F.weight_quant(w)
    del w
    qa = torch.empty((M, K), dtype=torch.uint8, device=dev)
    sa = torch.empty((M, K // 128), dtype=torch.float32, device=dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    torch.cuda.synchronize()
    return dict(M=M, N=N, K=K, x=x, qa=qa, sa=sa, qw=qw, sw=sw, y=y, F=F, desc=synth.PREFILL.desc)


def prefill_config(M, N, K, world):
    """The `config` of the headline line; the reference arm reports the same one (its
    bounded per-step sample is described in its cpu_baseline.sample)."""
    return {"workload": f"prefill-shaped linear: act_quant + block-scaled FP8 GEMM, M={M} N={N} K={K}, "
                        "128-ch act groups, 128x128 weight blocks, fp32 scales, bf16 out",
            "M_per_gpu": M, "N": N, "K": K, "parallelism": f"dp{world} (token batches)",
            "l2": "inputs larger than L2 (W 235 MB); no flush"}


def run_ours(args, world, rank, local):
    import torch
    import torch.distributed as dist
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    peaks, peak_src = load_peaks()
    if args.workload != "prefill":
        return run_other(args, world, rank, dev, peaks, peak_src)

    S = setup_prefill(dev, rank)
    F, M, N, K = S["F"], S["M"], S["N"], S["K"]
    stream = torch.cuda.current_stream()
    flops = 2.0 * M * N * K

    def step():
        F.fp8_act_quant(S["x"], S["qa"], S["sa"], stream=stream)
        F.fp8_block_gemm(S["qa"], S["sa"], S["qw"], S["sw"], S["y"], stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert F.fp8_device_error() == 0

    # -------- timed region: inputs resident in HBM
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t0.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            F.fp8_act_quant(S["x"], S["qa"], S["sa"], stream=stream)
            ev[i][1].record(stream)
            F.fp8_block_gemm(S["qa"], S["sa"], S["qw"], S["sw"], S["y"], stream=stream)
            ev[i][2].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = t0.elapsed_time(t1)
    aq_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    gm_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    assert F.fp8_device_error() == 0

    # -------- end to end through the public API with host buffers
    e2e_ms = e2e_pipelined(S, args.steps, max(1, args.warmup // 2), world)

    ms, e2e_ms, aq_ms, gm_ms = reduce_max([ms, e2e_ms, aq_ms, gm_ms], dev)

    tflops = weak_scaling_tflops(flops, world, args.steps, ms)
    e2e_tflops = weak_scaling_tflops(flops, world, args.steps, e2e_ms)
    gemm_tflops = flops / (gm_ms * 1e-3) / 1e12
    aq_bytes = M * K * 2 + M * K + M * (K // 128) * 4
    aq_gbs = aq_bytes / (aq_ms * 1e-3) / 1e9
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16
    # the power-capped figure (seconds of back-to-back GEMMs), for a GEMM timed inside
    # a long loop of steps; `frac` stays against the burst figure
    fp8_peak_sust = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * FP8_OVER_BF16

    out = {
        "metric": METRIC, "value": round(tflops, 2), "unit": "TFLOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
        "data": "synthetic (seeded N(0,1) activations with 1% outlier channels x20, N(0,0.02) weights)",
        "config": prefill_config(M, N, K, world),
        "gpu_launches": 2 * args.steps,
        "e2e": {"value": round(e2e_tflops, 2), "unit": "TFLOPS", "h2d_bytes_per_step": M * K * 2,
                "d2h_bytes_per_step": M * N * 2},
        "roofline": {"bound": "tensor", "kernel": "k_gemm_wide", "achieved": round(gemm_tflops, 1),
                     "peak": round(fp8_peak, 1), "unit": "TFLOP/s", "frac": round(gemm_tflops / fp8_peak, 4),
                     "peak_source": f"{peak_src} bf16 burst x {FP8_OVER_BF16} (nominal fp8/bf16 ratio)",
                     "traffic": profiled_traffic("k_gemm_wide prefill"),
                     "peak_sustained": round(fp8_peak_sust, 1),
                     "frac_vs_sustained": round(gemm_tflops / fp8_peak_sust, 4)},
        "act_quant": {"GB/s": round(aq_gbs, 1), "us": round(aq_ms * 1e3, 2), "bytes": aq_bytes,
                      "peak_GB/s": peaks["hbm_gbs"], "frac": round(aq_gbs / peaks["hbm_gbs"], 4),
                      "bound": "hbm", "peak_source": peak_src,
                      "traffic": profiled_traffic("k_act_quant prefill")},
        "gemm_us": round(gm_ms * 1e3, 2),
        "clocks": clk.summary(),
    }
    if world == 1 and not args.no_rows:
        out["rows"] = measure_rows(dev, peaks)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline_prefill(S, dev)
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def e2e_pipelined(S, steps, warm, world):
    """Every step copies its x from pinned host memory, quantises it and multiplies
    it (act_quant + GEMM on a compute stream) and copies y back to pinned host memory.  The
    copies run on their own streams with two device buffers each, so step i's
    copy-out and step i+2's copy-in overlap step i+1's kernels, as a serving loop
    would run them.  Returns the device time from the first copy-in to the last
    copy-out (ms)."""
    import torch
    import torch.distributed as dist
    F = S["F"]
    x_host = S["x"].cpu().pin_memory()
    y_host = [torch.empty(S["y"].shape, dtype=S["y"].dtype).pin_memory() for _ in range(2)]
    xd = [torch.empty_like(S["x"]) for _ in range(2)]
    yd = [torch.empty_like(S["y"]) for _ in range(2)]
    h2d, d2h, stream = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event(enable_timing=False)
    x_ready, x_free, y_ready, y_free = [ev(), ev()], [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def run(n):
        for b in range(2):
            x_free[b].record(stream)
            y_free[b].record(stream)
        for i in range(n):
            b = i & 1
            h2d.wait_event(x_free[b])
            with torch.cuda.stream(h2d):
                xd[b].copy_(x_host, non_blocking=True)
            x_ready[b].record(h2d)
            stream.wait_event(x_ready[b])
            stream.wait_event(y_free[b])
            F.fp8_act_quant(xd[b], S["qa"], S["sa"], stream=stream)
            x_free[b].record(stream)
            F.fp8_block_gemm(S["qa"], S["sa"], S["qw"], S["sw"], yd[b], stream=stream)
            y_ready[b].record(stream)
            d2h.wait_event(y_ready[b])
            with torch.cuda.stream(d2h):
                y_host[b].copy_(yd[b], non_blocking=True)
            y_free[b].record(d2h)

    run(warm)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(h2d)
    stream.wait_event(t0)
    d2h.wait_event(t0)
    run(steps)
    t1.record(d2h)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1)


def time_launches(fn, iters, warm=2):
    import torch
    for _ in range(warm):
        fn()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record()
    for _ in range(iters):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters


def time_graph(fn, iters, warm=2):
    """Device time per call of `fn` with `iters` calls captured in one CUDA graph and
    replayed: what a serving loop that launches through graphs sees, free of the
    Python / ctypes launch overhead that bounds microsecond-scale kernels eagerly."""
    import torch
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(iters):
            fn()
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    g.replay()
    b.record()
    torch.cuda.synchronize()
    del g
    return a.elapsed_time(b) / iters


def measure_rows(dev, peaks):
    """Every hot-path row on its own configuration (CUDA events, a few launches each)."""
    import torch
    import fp8_block_scaled_12_b200 as F
    import synth
    res = {}
    hbm = peaks["hbm_gbs"]
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16
    # act_quant sweep (per-128 fp32 and ue8m0) and per-tensor e4m3 / e5m2 at 16384 x 7168
    x = synth.activations(16384, 7168, seed=0, dist="t3", device=dev)
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.uint8, device=dev)
    s = torch.empty((M, K // 128), dtype=torch.float32, device=dev)
    s1 = torch.empty((1,), dtype=torch.float32, device=dev)
    for name, sf in (("act_quant_fp32", F.SCALE_FP32), ("act_quant_ue8m0", F.SCALE_UE8M0)):
        ms = time_launches(lambda: F.fp8_act_quant(x, q, s, scale_fmt=sf), 20)
        b = M * K * 3 + M * (K // 128) * 4
        res[name + " 16384x7168"] = {"GB/s": round(b / ms / 1e6, 1), "frac_hbm": round(b / ms / 1e6 / hbm, 4)}
    for name, fmt in (("per_tensor_e4m3", F.E4M3), ("per_tensor_e5m2", F.E5M2)):
        ms = time_launches(lambda: F.fp8_weight_quant(x, q, s1, block=0, fmt=fmt), 10)
        b = M * K * 3 + 4
        res[name + " 16384x7168"] = {"GB/s (algorithmic 3 B/elt)": round(b / ms / 1e6, 1),
                                      "frac_hbm": round(b / ms / 1e6 / hbm, 4)}
    # the smaller sweep tensors (1024 and 4096 rows; 1024 is launch-bound and reported,
    # not graded): each timed launch uses its own buffer set, with enough sets that the
    # data in flight exceeds the L2, so no launch finds its input there
    for Ms in (1024, 4096):
        nsets = max(2, -(-160 * 2 ** 20 // (Ms * K * 3)))
        sets = [(synth.activations(Ms, K, seed=i, dist="t3", device=dev),
                 torch.empty((Ms, K), dtype=torch.uint8, device=dev),
                 torch.empty((Ms, K // 128), dtype=torch.float32, device=dev),
                 torch.empty((1,), dtype=torch.float32, device=dev)) for i in range(nsets)]
        for name, sf in (("act_quant_fp32", F.SCALE_FP32), ("act_quant_ue8m0", F.SCALE_UE8M0)):
            turn = itertools.cycle(sets)

            def aq():
                xi, qi, si, _ = next(turn)
                F.fp8_act_quant(xi, qi, si, scale_fmt=sf)

            ms_e = time_launches(aq, 4 * nsets)
            ms = time_graph(aq, 4 * nsets)
            b = Ms * K * 3 + Ms * (K // 128) * 4
            res[f"{name} {Ms}x7168"] = {"GB/s": round(b / ms / 1e6, 1), "frac_hbm": round(b / ms / 1e6 / hbm, 4),
                                        "us": round(ms * 1e3, 2), "timing": "CUDA graph replay",
                                        "us_eager": round(ms_e * 1e3, 2)}
        for name, fmt in (("per_tensor_e4m3", F.E4M3), ("per_tensor_e5m2", F.E5M2)):
            turn = itertools.cycle(sets)

            def pt():
                xi, qi, _, s1i = next(turn)
                F.fp8_weight_quant(xi, qi, s1i, block=0, fmt=fmt)

            ms_e = time_launches(pt, 4 * nsets)
            ms = time_graph(pt, 4 * nsets)
            b = Ms * K * 3 + 4
            res[f"{name} {Ms}x7168"] = {"GB/s (algorithmic 3 B/elt)": round(b / ms / 1e6, 1),
                                        "frac_hbm": round(b / ms / 1e6 / hbm, 4), "us": round(ms * 1e3, 2),
                                        "timing": "CUDA graph replay", "us_eager": round(ms_e * 1e3, 2)}
        del sets
    # delayed scaling: one pass, previous step's scale, amax history of 16 (3 B/elt + state)
    ds = F.DelayedScaling(hist_len=16, device=dev)
    nclip = torch.empty(1, dtype=torch.int64, device=dev)
    sused = torch.empty(1, dtype=torch.float32, device=dev)
    ms = time_launches(lambda: F.fp8_delayed_quant(x, q, ds.scale, ds.pos, ds.history, nclip, sused), 20)
    b = M * K * 3
    res["delayed_scaling e4m3 16384x7168 (single pass)"] = {"GB/s (3 B/elt)": round(b / ms / 1e6, 1),
                                                            "frac_hbm": round(b / ms / 1e6 / hbm, 4),
                                                            "us": round(ms * 1e3, 2)}
    del x, q, s
    # weight_quant 128x128 on the prefill weight
    w = synth.weights(28672, 8192, 0.02, seed=0, device=dev)
    qw = torch.empty(w.shape, dtype=torch.uint8, device=dev)
    sw = torch.empty((224, 64), dtype=torch.float32, device=dev)
    ms = time_launches(lambda: F.fp8_weight_quant(w, qw, sw), 10)
    b = w.numel() * 3 + sw.numel() * 4
    res["weight_quant 28672x8192"] = {"GB/s": round(b / ms / 1e6, 1), "frac_hbm": round(b / ms / 1e6 / hbm, 4)}
    del w, qw, sw
    # decode GEMM, ue8m0, M in {1, 8, 32, 64}; launches alternate between two weight
    # copies (2 x 132 MB, above the L2) so no launch finds its weights in L2
    wds = []
    for c in range(2):
        wd = synth.weights(18432, 7168, 0.015, seed=c, device=dev)
        wds.append(F.weight_quant(wd, scale_fmt=F.SCALE_UE8M0))
        del wd
    swd = wds[0][1]
    for Md in (1, 8, 32, 64):
        xd = synth.activations(Md, 7168, seed=0, device=dev)
        qa, sa = F.act_quant(xd, scale_fmt=F.SCALE_UE8M0)
        y = torch.empty((Md, 18432), dtype=torch.bfloat16, device=dev)
        turn = itertools.cycle(wds)

        def dgemm():
            qwd, swd_ = next(turn)
            F.fp8_block_gemm(qa, sa, qwd, swd_, y)

        ms = time_launches(dgemm, 20)
        ms_g = time_graph(dgemm, 20)
        b = 18432 * 7168 + swd.numel() * 4 + Md * (7168 + 56 * 4 + 18432 * 2)
        res[f"decode_gemm M={Md}"] = {"us": round(ms * 1e3, 2), "GB/s": round(b / ms / 1e6, 1),
                                      "frac_hbm": round(b / ms / 1e6 / hbm, 4),
                                      "TFLOPS": round(2 * Md * 18432 * 7168 / ms / 1e9, 2),
                                      "us_graph": round(ms_g * 1e3, 2), "frac_hbm_graph": round(b / ms_g / 1e6 / hbm, 4)}
    del wds, swd
    # grouped MoE GEMM
    p = synth.MOE.params
    row_token, _, off = synth.routing(p["T"], p["E"], p["topk"], seed=0)
    xt = synth.activations(p["T"], p["K"], seed=0, device=dev)
    qa, sa = F.act_quant(xt[row_token.to(dev)])
    E, N, K = p["E"], p["N"], p["K"]
    qwe = torch.empty((E, N, K), dtype=torch.uint8, device=dev)
    swe = torch.empty((E, N // 128, K // 128), dtype=torch.float32, device=dev)
    for e in range(E):
        F.fp8_weight_quant(synth.weights(N, K, p["w_std"], seed=0, chunk=e, device=dev), qwe[e], swe[e])
    y = torch.empty((qa.shape[0], N), dtype=torch.bfloat16, device=dev)
    offd = off.to(dev)
    # fused MoE layer: device routing of seeded scores, act_quant of the 4096 tokens,
    # expert GEMMs gathering their rows and adding gate-weighted outputs per token
    g = torch.Generator(device=dev).manual_seed(3)
    scores = torch.rand((p["T"], E), generator=g, device=dev, dtype=torch.float32)
    route = F.moe_route(scores, p["topk"])
    qt, st_ = F.act_quant_permute(xt, route)
    out = torch.empty((p["T"], N), dtype=torch.float32, device=dev)

    def moe_step():
        F.fp8_moe_route(scores, p["topk"], route["ids"], route["w"], route["offsets"], route["row_token"],
                        route["row_weight"], route["token_row"], route["workspace"])
        F.fp8_act_quant_permute(xt, route, qt, st_)
        F.fp8_moe_gemm(qt, st_, qwe, swe, route, out)

    ms_f = time_launches(moe_step, 5)
    ms_r = time_launches(lambda: F.fp8_moe_route(scores, p["topk"], route["ids"], route["w"], route["offsets"],
                                                 route["row_token"], route["row_weight"], route["token_row"],
                                                 route["workspace"]), 10)
    fl_m = 2.0 * p["T"] * p["topk"] * N * K
    res["moe layer (route + act_quant_permute + GEMM with weighted scatter) 4096 tok top-8/256"] = {
        "us": round(ms_f * 1e3, 1), "TFLOPS": round(fl_m / ms_f / 1e9, 1), "route_us": round(ms_r * 1e3, 1)}
    del out, route, scores
    ms = time_launches(lambda: F.fp8_grouped_gemm(qa, sa, qwe, swe, offd, y), 5)
    fl = 2.0 * qa.shape[0] * N * K
    b = qwe.numel() + swe.numel() * 4 + qa.numel() + sa.numel() * 4 + y.numel() * 2
    res["grouped_gemm moe 32768x2048x7168 E=256"] = {"us": round(ms * 1e3, 1),
                                                    "TFLOPS": round(fl / ms / 1e9, 1),
                                                    "frac_fp8_peak": round(fl / ms / 1e9 / fp8_peak, 4),
                                                    "GB/s": round(b / ms / 1e6, 1),
                                                    "frac_hbm": round(b / ms / 1e6 / hbm, 4)}
    assert F.fp8_device_error() == 0
    del qwe, swe, qa, sa, y
    res.update(measure_fused_rows(dev, peaks))
    res.update(measure_mx_rows(dev, peaks))
    return res


def measure_fused_rows(dev, peaks):
    """Steps beside the GEMM: the BF16 path's weight dequantisation, and the prefill GEMM
    whose epilogue quantises its output for the next layer (no separate act_quant pass)."""
    import torch
    import fp8_block_scaled_12_b200 as F
    import synth
    res = {}
    hbm = peaks["hbm_gbs"]
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16
    p = synth.PREFILL.params
    M, N, K = p["M"], p["N"], p["K"]
    w = synth.weights(N, K, p["w_std"], seed=0, device=dev)
    qw, sw = F.weight_quant(w)
    wb = torch.empty_like(w)
    ms = time_launches(lambda: F.fp8_weight_dequant(qw, sw, wb), 10)
    b = N * K * 3 + sw.numel() * 4
    res["weight_dequant 28672x8192"] = {"GB/s": round(b / ms / 1e6, 1), "frac_hbm": round(b / ms / 1e6 / hbm, 4),
                                        "us": round(ms * 1e3, 1)}
    del w, wb
    x = synth.activations(M, K, seed=0, device=dev)
    qa, sa = F.act_quant(x)
    qy = torch.empty((M, N), dtype=torch.uint8, device=dev)
    sy = torch.empty((M, N // 128), dtype=torch.float32, device=dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    fl = 2.0 * M * N * K
    ms = time_launches(lambda: F.fp8_block_gemm_quant(qa, sa, qw, sw, qy, sy), 10)
    res["block_gemm_quant prefill 4096x28672x8192 (codes + scales out, no y)"] = {
        "us": round(ms * 1e3, 1), "TFLOPS": round(fl / ms / 1e9, 1), "frac_fp8_peak": round(fl / ms / 1e9 / fp8_peak, 4)}
    ms = time_launches(lambda: F.fp8_block_gemm_quant(qa, sa, qw, sw, qy, sy, y), 10)
    res["block_gemm_quant prefill 4096x28672x8192 (y, codes and scales out)"] = {
        "us": round(ms * 1e3, 1), "TFLOPS": round(fl / ms / 1e9, 1), "frac_fp8_peak": round(fl / ms / 1e9 / fp8_peak, 4)}
    assert F.fp8_device_error() == 0
    return res


def measure_mx_rows(dev, peaks):
    """The tensor core's scale path: MXFP8 quantisation and GEMM (32-element E8M0
    blocks), and the ue8m0 (power-of-two) configurations on it."""
    import torch
    import fp8_block_scaled_12_b200 as F
    import synth
    res = {}
    hbm = peaks["hbm_gbs"]
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16
    x = synth.activations(16384, 7168, seed=0, dist="t3", device=dev)
    q = torch.empty(x.shape, dtype=torch.uint8, device=dev)
    e8 = torch.empty((F.mx_sf_bytes(16384, 7168),), dtype=torch.uint8, device=dev)
    ms = time_launches(lambda: F.fp8_mx_quant(x, q, e8), 20)
    b = x.numel() * 3 + x.numel() // 32
    res["mx_quant 16384x7168"] = {"GB/s": round(b / ms / 1e6, 1), "frac_hbm": round(b / ms / 1e6 / hbm, 4)}
    del x, q, e8
    # prefill shape: MXFP8 (32-element exponents) and the ue8m0 scales (128 / 128x128) packed
    p = synth.PREFILL.params
    M, N, K = p["M"], p["N"], p["K"]
    xa = synth.activations(M, K, seed=0, device=dev)
    w = synth.weights(N, K, p["w_std"], seed=0, device=dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    fl = 2.0 * M * N * K
    qa, ea = F.mx_quant(xa)
    qw, ew = F.mx_quant(w)
    ms = time_launches(lambda: F.fp8_mx_gemm(qa, ea, qw, ew, y), 10)
    res["mx_gemm e8m0x32 prefill 4096x28672x8192"] = {"us": round(ms * 1e3, 1), "TFLOPS": round(fl / ms / 1e9, 1),
                                                       "frac_fp8_peak": round(fl / ms / 1e9 / fp8_peak, 4)}
    qa, sa = F.act_quant(xa, scale_fmt=F.SCALE_UE8M0)
    qw, sw = F.weight_quant(w, scale_fmt=F.SCALE_UE8M0)
    del w
    ew = F.mx_pack_pow2(sw, N, K, 128)                       # weights: once
    ea = torch.empty((F.mx_sf_bytes(M, K),), dtype=torch.uint8, device=dev)

    def pow2_step():                                         # activations: every call
        F.fp8_mx_pack_pow2(sa, M, K, 1, ea)
        F.fp8_mx_gemm(qa, ea, qw, ew, y)

    ms = time_launches(pow2_step, 10)
    res["mx_gemm ue8m0 prefill 4096x28672x8192 (pack + gemm)"] = {
        "us": round(ms * 1e3, 1), "TFLOPS": round(fl / ms / 1e9, 1), "frac_fp8_peak": round(fl / ms / 1e9 / fp8_peak, 4)}
    ms = time_launches(lambda: F.fp8_block_gemm(qa, sa, qw, sw, y), 10)
    res["block_gemm (promotion) ue8m0 prefill 4096x28672x8192"] = {
        "us": round(ms * 1e3, 1), "TFLOPS": round(fl / ms / 1e9, 1), "frac_fp8_peak": round(fl / ms / 1e9 / fp8_peak, 4)}
    del qa, sa, qw, sw, xa, y, ea, ew
    # decode config (ue8m0) on the scale path: weights packed once, activations per call
    # (two weight copies alternated, as for the promotion decode rows)
    wds = []
    for c in range(2):
        wd = synth.weights(18432, 7168, 0.015, seed=c, device=dev)
        qwd, swd = F.weight_quant(wd, scale_fmt=F.SCALE_UE8M0)
        del wd
        wds.append((qwd, F.mx_pack_pow2(swd, 18432, 7168, 128)))
    ewd = wds[0][1]
    for Md in (1, 64):
        xd = synth.activations(Md, 7168, seed=0, device=dev)
        qa, sa = F.act_quant(xd, scale_fmt=F.SCALE_UE8M0)
        ea = torch.empty((F.mx_sf_bytes(Md, 7168),), dtype=torch.uint8, device=dev)
        y = torch.empty((Md, 18432), dtype=torch.bfloat16, device=dev)
        turn = itertools.cycle(wds)

        def dstep():
            qwd, ewd_ = next(turn)
            F.fp8_mx_pack_pow2(sa, Md, 7168, 1, ea)
            F.fp8_mx_gemm(qa, ea, qwd, ewd_, y)

        ms = time_launches(dstep, 20)
        b = 18432 * 7168 + ewd.numel() + Md * (7168 + 56 * 4 + 18432 * 2)
        res[f"mx_gemm ue8m0 decode M={Md} (pack + gemm)"] = {"us": round(ms * 1e3, 2), "GB/s": round(b / ms / 1e6, 1),
                                                            "frac_hbm": round(b / ms / 1e6 / hbm, 4)}
    del wds
    # decode on MXFP8 operands (E8M0 per 32 elements on both sides), two weight copies
    wms = []
    for c in range(2):
        wd = synth.weights(18432, 7168, 0.015, seed=c, device=dev)
        wms.append(F.mx_quant(wd))
        del wd
    for Md in (1, 64):
        xd = synth.activations(Md, 7168, seed=0, device=dev)
        qa, ea = F.mx_quant(xd)
        y = torch.empty((Md, 18432), dtype=torch.bfloat16, device=dev)
        turn = itertools.cycle(wms)

        def mstep():
            qwm, ewm = next(turn)
            F.fp8_mx_gemm(qa, ea, qwm, ewm, y)

        ms = time_launches(mstep, 20)
        ms_g = time_graph(mstep, 20)
        b = 18432 * 7168 + wms[0][1].numel() + Md * (7168 + 7168 // 32 + 18432 * 2)
        res[f"mx_gemm e8m0x32 decode M={Md}"] = {"us": round(ms * 1e3, 2), "GB/s": round(b / ms / 1e6, 1),
                                               "frac_hbm": round(b / ms / 1e6 / hbm, 4),
                                               "us_graph": round(ms_g * 1e3, 2),
                                               "frac_hbm_graph": round(b / ms_g / 1e6 / hbm, 4)}
    assert F.fp8_device_error() == 0
    return res


def host_cores():
    """(cores this process may run on, cores the host reports)."""
    try:
        usable = len(os.sched_getaffinity(0))
    except AttributeError:
        usable = os.cpu_count() or 1
    return usable, os.cpu_count() or usable


def cpu_baseline_prefill(S, dev):
    """The oracle as it stands (plain C, fp64 GEMM) on bounded samples of the workloads,
    on the host cores (about 10 s of host time on a 16-core host):
      - GEMM: a few prefill rows against all 28672 weight rows, single-threaded and
        split over every usable core; full-size times are extrapolated from the
        measured fp64 MAC/s (labelled as such);
      - act_quant: a 4096 x 7168 sweep tensor single-threaded and the full 16384 x 7168
        sweep tensor over every usable core (Student-t(3) entries, fp32 scales)."""
    import oracle as O
    import synth
    K, N, M = S["K"], S["N"], S["M"]
    usable, reported = host_cores()
    qw = S["qw"].cpu().numpy()
    sw = S["sw"].cpu().numpy()
    rows_mt = 16 * usable                 # about 10 s of work on every core
    x = S["x"][:rows_mt].cpu()
    qa, sa = O.act_quant(x)

    t = time.perf_counter()
    O.gemm_rows(qa, sa, qw, sw, rows=[0, 1, 2])
    t1 = time.perf_counter() - t
    mac1 = 3 * N * K / t1
    t = time.perf_counter()
    O.gemm_rows(qa, sa, qw, sw, rows=list(range(rows_mt)), threads=usable)
    tmt = time.perf_counter() - t
    macmt = rows_mt * N * K / tmt
    full_mac = float(M) * N * K

    xs = synth.activations(16384, 7168, seed=0, dist="t3", device=dev).cpu()
    aq_bytes = lambda m: m * 7168 * 3 + m * 56 * 4
    t = time.perf_counter()
    O.act_quant(xs[:4096])
    taq1 = time.perf_counter() - t
    t = time.perf_counter()
    O.act_quant(xs, threads=usable)
    taqmt = time.perf_counter() - t
    return {"value": round(2.0 * macmt / 1e12, 6), "unit": "TFLOPS", "cores": usable, "kind": "oracle",
            "host_cores": reported,
            "sample": f"fp64 GEMM of {rows_mt} prefill rows x {N} x {K} split over {usable} threads "
                      f"(plus 3 rows single-threaded); act_quant of the 16384x7168 sweep tensor over {usable} "
                      f"threads and of 4096x7168 single-threaded",
            "gemm": {"mac_per_s_1thread": round(mac1), "mac_per_s_all_cores": round(macmt),
                     "prefill_full_s_extrapolated_1thread": round(full_mac / mac1, 1),
                     "prefill_full_s_extrapolated_all_cores": round(full_mac / macmt, 1),
                     "TFLOPS_1thread": round(2.0 * mac1 / 1e12, 6)},
            "act_quant": {"GB/s_1thread (4096x7168)": round(aq_bytes(4096) / taq1 / 1e9, 3),
                          "GB/s_all_cores (16384x7168)": round(aq_bytes(16384) / taqmt / 1e9, 3),
                          "s_all_cores (16384x7168)": round(taqmt, 2)},
            "seconds": round(t1 + tmt + taq1 + taqmt, 2)}


def run_other(args, world, rank, dev, peaks, peak_src):
    """Secondary workloads: one JSON line each (not the headline)."""
    import torch
    out = {"metric": METRIC, "workload": args.workload, "n_gpus": world}
    out["rows"] = measure_rows(dev, peaks)
    if rank == 0:
        print(json.dumps(out), flush=True)


# ------------------------------------------------------------- reference arm
def run_reference(args, world, rank):
    """The CPU oracle on the prefill workload's shapes, on every usable host core: each
    step quantises one activation row and computes its fp64 GEMM against all 28672
    weight rows (a bounded sample of the step; the rows are split over the threads)."""
    if rank != 0:
        return
    import oracle as O
    import synth
    p = synth.PREFILL.params
    M, N, K = p["M"], p["N"], p["K"]
    usable, reported = host_cores()
    ch = synth.outlier_channels(K, synth.n_outliers(K, p["outlier_frac"]), seed=0)
    x = synth.activations(4, K, seed=0, outliers=ch, factor=p["factor"])
    w = synth.weights(N, K, p["w_std"], seed=0)
    qw, sw = O.weight_quant(w, threads=usable)
    del w
    # one row against all weight rows: the weight rows are split into per-thread slices
    # on 128-row block boundaries (each slice keeps its own block scales)
    slices = O._split(N, usable, 128)

    def step():
        qa, sa = O.act_quant(x[:1])
        O._run_parallel(lambda a, b: O.gemm_rows(qa, sa, qw[a:b], sw[a // 128:(b + 127) // 128]),
                        slices, usable)

    for _ in range(args.warmup):
        step()
    t = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t
    fl = 2.0 * N * K * args.steps
    v = fl / dt / 1e12
    out = {"impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": "TFLOPS", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3 / args.steps, 2),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "config": prefill_config(M, N, K, world),
           "cpu_baseline": {"value": round(v, 6), "unit": "TFLOPS", "cores": usable, "host_cores": reported,
                            "kind": "oracle",
                            "sample": f"act_quant of 1 row + fp64 GEMM of 1 row x {N} x {K} per step, "
                                      f"weight rows split over {usable} threads"},
           "e2e": {"value": round(v, 6), "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["prefill", "decode", "moe", "sweep"], default="prefill")
    ap.add_argument("--no-rows", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    world, rank, local = dist_setup()
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
