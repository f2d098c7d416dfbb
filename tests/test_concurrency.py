"""Concurrent use of the library: the C ABI keeps no per-call state (its only host-side
state is set-up caches guarded for concurrent use), so two host threads driving their
own streams at the same time -- quantise, block GEMM, MXFP8 GEMM and a routed MoE layer,
each on its own buffers -- must produce exactly what the same calls produce one after
another."""
import threading

import pytest
import torch

import fp8_block_scaled_12_b200 as F
import synth

pytestmark = pytest.mark.gpu


def make_work(dev, seed):
    x = synth.activations(300, 1024, seed=seed, device=dev)
    w = synth.weights(768, 1024, 0.02, seed=seed, device=dev)
    xd = synth.activations(40, 1024, seed=seed + 1, device=dev)
    E, k = 8, 2
    g = torch.Generator(device=dev).manual_seed(seed)
    scores = torch.rand((200, E), generator=g, device=dev)
    xt = synth.activations(200, 1024, seed=seed + 2, device=dev)
    qwe = torch.empty((E, 256, 1024), dtype=torch.uint8, device=dev)
    swe = torch.empty((E, 2, 8), dtype=torch.float32, device=dev)
    for e in range(E):
        F.fp8_weight_quant(synth.weights(256, 1024, 0.02, seed=seed, chunk=e, device=dev), qwe[e], swe[e])
    torch.cuda.synchronize()

    def run(stream):
        with torch.cuda.stream(stream):
            qa, sa = F.act_quant(x, stream=stream)
            qw, sw = F.weight_quant(w, stream=stream)
            y = F.block_gemm(qa, sa, qw, sw, stream=stream)
            qd, sd = F.act_quant(xd, stream=stream)
            yd = F.block_gemm(qd, sd, qw, sw, out_dtype=torch.float32, stream=stream)
            qm, em = F.mx_quant(x, stream=stream)
            qmw, emw = F.mx_quant(w, stream=stream)
            ym = F.mx_gemm(qm, em, qmw, emw, stream=stream)
            r = F.moe_route(scores, k, stream=stream)
            qs, ss = F.act_quant_permute(xt, r, stream=stream)
            routed = [r[n] for n in ("ids", "w", "offsets", "row_token", "row_weight", "token_row")]
        # (the E8M0 buffers em / emw also hold the slots of padding rows, which nothing
        # writes; the exponents that matter are checked through ym)
        return [qa, sa, qw, sw, y, qd, sd, yd, qm, qmw, ym, qs, ss] + routed

    return run


def test_two_threads_two_streams(cuda_device):
    works = [make_work(cuda_device, s) for s in (1, 2)]
    streams = [torch.cuda.Stream() for _ in works]
    ref = []
    for wk, st in zip(works, streams):
        ref.append([t.clone() for t in wk(st)])
        torch.cuda.synchronize()
    for rep in range(3):
        outs = [None, None]
        errors = []

        def worker(i):
            try:
                torch.cuda.set_device(cuda_device)
                res = None
                for _ in range(4):              # several rounds so the two streams overlap
                    res = works[i](streams[i])
                outs[i] = res
            except Exception as e:             # surfaced below
                errors.append(e)

        th = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
        for t in th:
            t.start()
        for t in th:
            t.join()
        assert not errors, errors
        torch.cuda.synchronize()
        assert F.fp8_device_error() == 0
        for i in range(2):
            for j, (got, exp) in enumerate(zip(outs[i], ref[i])):
                assert torch.equal(got.view(torch.uint8), exp.view(torch.uint8)), f"thread {i} output {j} rep {rep}"
