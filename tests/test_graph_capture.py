"""The library's kernels inside CUDA graphs.

Every kernel is launched with programmatic stream serialisation (it may start while
its predecessor finishes and waits for it before touching operand data).  Captured
into a CUDA graph those launches become programmatic dependency edges; replaying the
graph must give exactly what the same calls give eagerly.  Covered: the prefill-shaped
step (act_quant + block GEMM), a decode step on the weight-stationary kernel, the
MXFP8 GEMM, and the routed MoE layer (routing kernels, permuted act_quant, a memset and
the grouped GEMM with its scatter-add)."""
import pytest
import torch

import fp8_block_scaled_12_b200 as F
import synth

pytestmark = pytest.mark.gpu


def replay_equals_eager(step, outputs, replays=3):
    """Run `step` eagerly, keep its outputs, capture it, replay it `replays` times
    after scribbling over the outputs, and compare bit for bit."""
    step()
    torch.cuda.synchronize()
    ref = [o.clone() for o in outputs]
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()                                  # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        step()
    for _ in range(replays):
        for o in outputs:
            o.view(torch.uint8).fill_(0xA5)
        g.replay()
        torch.cuda.synchronize()
        assert F.fp8_device_error() == 0
        for o, r in zip(outputs, ref):
            assert torch.equal(o.view(torch.uint8), r.view(torch.uint8))
    del g


def test_prefill_and_decode_steps_in_a_graph(cuda_device):
    dev = cuda_device
    w = synth.weights(2304, 2048, 0.02, seed=1, device=dev)
    qw, sw = F.weight_quant(w)
    for M in (1000, 40):                        # 128 x 256 tiles; weight-stationary
        x = synth.activations(M, 2048, seed=M, device=dev)
        qa = torch.empty((M, 2048), dtype=torch.uint8, device=dev)
        sa = torch.empty((M, 16), dtype=torch.float32, device=dev)
        y = torch.empty((M, 2304), dtype=torch.bfloat16, device=dev)

        def step():
            F.fp8_act_quant(x, qa, sa)
            F.fp8_block_gemm(qa, sa, qw, sw, y)

        replay_equals_eager(step, [qa, sa, y])


def test_mx_gemm_in_a_graph(cuda_device):
    dev = cuda_device
    w = synth.weights(1024, 1024, 0.02, seed=2, device=dev)
    x = synth.activations(64, 1024, seed=2, device=dev)
    qw, ew = F.mx_quant(w)
    qa = torch.empty((64, 1024), dtype=torch.uint8, device=dev)
    ea = torch.empty((F.mx_sf_bytes(64, 1024),), dtype=torch.uint8, device=dev)
    y = torch.empty((64, 1024), dtype=torch.bfloat16, device=dev)

    def step():
        F.fp8_mx_quant(x, qa, ea)
        F.fp8_mx_gemm(qa, ea, qw, ew, y)

    # (ea's atom also holds the exponent slots of rows 64-127, which nothing writes, so
    # it is checked through y rather than scribbled over)
    replay_equals_eager(step, [qa, y])


def test_moe_layer_in_a_graph(cuda_device):
    dev = cuda_device
    T, E, k, N, K = 600, 16, 4, 256, 1024
    g = torch.Generator(device=dev).manual_seed(4)
    scores = torch.rand((T, E), generator=g, device=dev)
    x = synth.activations(T, K, seed=4, device=dev)
    qw = torch.empty((E, N, K), dtype=torch.uint8, device=dev)
    sw = torch.empty((E, N // 128, K // 128), dtype=torch.float32, device=dev)
    for e in range(E):
        F.fp8_weight_quant(synth.weights(N, K, 0.02, seed=4, chunk=e, device=dev), qw[e], sw[e])
    r = F.moe_route(scores, k)
    qs, ss = F.act_quant_permute(x, r)
    out = torch.empty((T, N), dtype=torch.float32, device=dev)

    def step():
        F.fp8_moe_route(scores, k, r["ids"], r["w"], r["offsets"], r["row_token"], r["row_weight"],
                        r["token_row"], r["workspace"])
        F.fp8_act_quant_permute(x, r, qs, ss)
        F.fp8_moe_gemm(qs, ss, qw, sw, r, out)

    # the scatter-add makes the output's last bits depend on the order of the fp32
    # additions, so the routing, permutation and quantised rows are compared exactly
    # and the output within the combine tolerance of its eager value
    step()
    torch.cuda.synchronize()
    ref_out = out.clone()
    replay_equals_eager(step, [r["ids"], r["w"], r["offsets"], r["row_token"], r["row_weight"], r["token_row"],
                               qs, ss])
    scale = ref_out.abs().max().item()
    assert torch.allclose(out, ref_out, rtol=0, atol=1e-5 * scale + 1e-30)
