import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size parity case")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def pytest_terminal_summary(terminalreporter):
    """List, per bf16 comparison, how many elements passed only through the heavy-
    cancellation allowance (beyond 1 bf16 ulp, within 1e-5 * sum|a w| + half an ulp)."""
    try:
        from _parity import ALLOWANCE_LOG
    except Exception:
        return
    if not ALLOWANCE_LOG:
        return
    tr = terminalreporter
    tr.section("bf16 cancellation allowance")
    total = sum(n for _, n, _ in ALLOWANCE_LOG)
    elems = sum(c for _, _, c in ALLOWANCE_LOG)
    tr.write_line(f"{total} of {elems} compared bf16 elements needed the allowance "
                  f"({len(ALLOWANCE_LOG)} comparisons)")
    for what, n, c in ALLOWANCE_LOG:
        if n:
            tr.write_line(f"  {what}: {n} of {c}")
