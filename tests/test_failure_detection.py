"""Failure detection without a GPU fault.

Every pipelined wait in the GEMM kernels is an mbarrier wait bounded in wall time;
when it runs out the kernel records FP8_ERR_TIMEOUT in a device-side error word and
returns instead of hanging.  The diagnostic entry point runs that same wait on a
barrier nothing ever arrives on, with a short limit, so the path is exercised here:
the status reaches the host, is cleared by reading it, and the context keeps
working.  A second diagnostic lowers the GEMM kernels' own wait limit to 1 ns so that
every GEMM kernel takes its abort path (drain the loads and MMAs in flight, free
tensor memory, return) -- run in a child process, then compared bit for bit with the
same calls at the normal limit.  Host-side failures (bad arguments) are covered by
test_abi_host.py.
"""
import os
import subprocess
import sys

import pytest
import torch

import fp8_block_scaled_12_b200 as F
import oracle as O
import synth
from _parity import check_fp32, codes

TIMEOUT = 6


def test_selftest_rejects_bad_limits():
    assert F.lib.fp8_selftest_bounded_wait(0, None) == 1
    assert F.lib.fp8_selftest_bounded_wait(-5, None) == 1
    assert F.lib.fp8_selftest_bounded_wait(20_000_000_000, None) == 1
    assert F.lib.fp8_set_wait_limit_ns(-1) == 1
    assert F.lib.fp8_set_wait_limit_ns(20_000_000_000) == 1


@pytest.mark.gpu
def test_gemm_abort_path_drains_and_recovers(cuda_device):
    child = os.path.join(os.path.dirname(os.path.abspath(__file__)), "abort_child.py")
    r = subprocess.run([sys.executable, child], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.strip().endswith("OK"), r.stdout[-2000:] + r.stderr[-4000:]


@pytest.mark.gpu
def test_bounded_wait_reports_timeout_and_context_survives(cuda_device):
    assert F.fp8_device_error() == 0
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    F.fp8_selftest_bounded_wait(50_000_000)        # 50 ms
    b.record()
    assert F.fp8_device_error() == TIMEOUT
    ms = a.elapsed_time(b)
    assert 40.0 <= ms < 2000.0, ms
    assert F.fp8_device_error() == 0              # reading cleared it
    # the context is intact: a quantise + GEMM afterwards is correct
    x = synth.activations(40, 512, seed=3)
    w = synth.weights(256, 512, 0.02, seed=3)
    qa, sa = F.act_quant(x.to(cuda_device))
    qw, sw = F.weight_quant(w.to(cuda_device))
    y = F.block_gemm(qa, sa, qw, sw, out_dtype=torch.float32)
    assert F.fp8_device_error() == 0
    y_ref, bound = O.gemm_rows(codes(qa), sa.cpu().numpy(), codes(qw), sw.cpu().numpy())
    check_fp32(y.cpu().numpy(), y_ref, bound, "after timeout")
