"""Child process of test_failure_detection.py::test_gemm_abort_path_drains_and_recovers.

Runs every GEMM kernel once with its pipeline waits limited to 1 ns, so each CTA gives
up at its first wait that does not succeed at once and takes the abort path (the
producer waits for the loads it issued, each issuer for its MMAs, then tensor memory is
freed).  Checks that every such call reports FP8_ERR_TIMEOUT, then restores the
limit and checks that the same calls reproduce, bit for bit, the outputs they gave
before.  Runs in its own process so nothing it does can disturb the other tests'
CUDA context.  Prints OK and exits 0 on success."""
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import fp8_block_scaled_12_b200 as F  # noqa: E402
import synth  # noqa: E402

TIMEOUT = 6


def main():
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    cases = {}
    # wide promotion kernel (M > 160), 8 x 14 tiles
    x = synth.activations(1024, 2048, seed=1, device=dev)
    w = synth.weights(3584, 2048, 0.02, seed=1, device=dev)
    qa, sa = F.act_quant(x)
    qw, sw = F.weight_quant(w)
    yw = torch.empty((1024, 3584), dtype=torch.bfloat16, device=dev)
    cases["wide"] = (lambda: F.fp8_block_gemm(qa, sa, qw, sw, yw), yw)
    # weight-stationary promotion kernel (decode)
    xd = synth.activations(40, 2048, seed=2, device=dev)
    qd, sd = F.act_quant(xd)
    yd = torch.empty((40, 3584), dtype=torch.float32, device=dev)
    cases["swap"] = (lambda: F.fp8_block_gemm(qd, sd, qw, sw, yd), yd)
    # MXFP8 kernels, wide and weight-stationary (two issuers)
    qmw, emw = F.mx_quant(w)
    qma, ema = F.mx_quant(x)
    ym = torch.empty((1024, 3584), dtype=torch.bfloat16, device=dev)
    cases["mx wide"] = (lambda: F.fp8_mx_gemm(qma, ema, qmw, emw, ym), ym)
    qmd, emd = F.mx_quant(xd)
    ymd = torch.empty((40, 3584), dtype=torch.bfloat16, device=dev)
    cases["mx swap"] = (lambda: F.fp8_mx_gemm(qmd, emd, qmw, emw, ymd), ymd)

    ref = {}
    for name, (fn, y) in cases.items():
        fn()
        torch.cuda.synchronize()
        assert F.fp8_device_error() == 0, name
        ref[name] = y.clone()
    F.fp8_set_wait_limit_ns(1)
    try:
        for name, (fn, y) in cases.items():
            fn()
            status = F.fp8_device_error()
            assert status == TIMEOUT, f"{name}: status {status} with a 1 ns wait limit"
    finally:
        F.fp8_set_wait_limit_ns(0)
    for name, (fn, y) in cases.items():
        y.zero_()
        fn()
        torch.cuda.synchronize()
        assert F.fp8_device_error() == 0, name
        assert torch.equal(y.view(torch.uint8), ref[name].view(torch.uint8)), f"{name}: output changed after abort"
    print("OK")


if __name__ == "__main__":
    main()
