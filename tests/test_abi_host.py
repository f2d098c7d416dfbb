"""Host-only checks of the C ABI: the library loads, exports every function the
header declares, and rejects bad arguments with the documented status before
touching the GPU (every call below fails validation, so nothing is launched)."""
import ctypes
import os
import re

import pytest

import fp8_block_scaled_12_b200 as F

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8lin.h")

OK, INVALID, SHAPE, ALIGN, UNSUP, CUDA, TIMEOUT, BADSCALE = range(8)
FAKE = 0x7F0000000000       # 16-byte aligned, never dereferenced
S = None                    # default stream


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fp8_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_four_operations():
    names = declared_functions()
    for n in ("fp8_act_quant", "fp8_weight_quant", "fp8_block_gemm", "fp8_grouped_gemm"):
        assert n in names


def test_library_exports_every_declared_function():
    lib = ctypes.CDLL(F.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_status_strings():
    assert F.fp8_status_string(OK) == "ok"
    for c in range(1, 8):
        assert F.fp8_status_string(c) not in ("ok", "unknown status")
    assert F.fp8_status_string(99) == "unknown status"


def aq(*a):
    return F.lib.fp8_act_quant(*a)


def test_act_quant_validation():
    # (x, M, K, ldx, group, fmt, sf, q, s, stream)
    assert aq(FAKE, -1, 128, 128, 128, 0, 0, FAKE, FAKE, S) == INVALID
    assert aq(FAKE, 4, 128, 64, 128, 0, 0, FAKE, FAKE, S) == INVALID        # ldx < K
    assert aq(FAKE, 4, 128, 128, 128, 2, 0, FAKE, FAKE, S) == INVALID       # bad format
    assert aq(FAKE, 4, 128, 128, 128, 0, 7, FAKE, FAKE, S) == INVALID       # bad scale format
    assert aq(FAKE, 4, 128, 128, 32, 0, 0, FAKE, FAKE, S) == UNSUP          # 32-element blocks: fp8_mx_quant
    assert aq(FAKE, 4, 136, 136, 128, 0, 0, FAKE, FAKE, S) == SHAPE         # K % 16
    assert aq(None, 4, 128, 128, 128, 0, 0, FAKE, FAKE, S) == INVALID       # null x
    assert aq(FAKE + 8, 4, 128, 128, 128, 0, 0, FAKE, FAKE, S) == ALIGN     # x not 16-byte aligned
    assert aq(FAKE, 4, 128, 132, 128, 0, 0, FAKE, FAKE, S) == ALIGN         # ldx % 8
    assert aq(FAKE, 0, 128, 128, 128, 0, 0, None, None, S) == OK            # M == 0: no-op


def test_weight_quant_validation():
    wq = F.lib.fp8_weight_quant
    assert wq(FAKE, 256, 256, 64, 0, 0, FAKE, FAKE, S) == UNSUP             # block 64 not built
    assert wq(FAKE, 256, 250, 128, 0, 0, FAKE, FAKE, S) == SHAPE
    assert wq(FAKE, 256, 256, 128, 0, 0, FAKE, None, S) == INVALID
    assert wq(FAKE, 256, 256, 128, 0, 0, FAKE + 4, FAKE, S) == ALIGN
    assert wq(FAKE, 0, 256, 0, 1, 0, None, None, S) == OK


def test_gemm_validation():
    g = F.lib.fp8_block_gemm
    # (qa, sa, qw, sw, M, N, K, out, y, stream)
    assert g(FAKE, FAKE, FAKE, FAKE, 16, 256, 200, 0, FAKE, S) == SHAPE     # K % 128
    assert g(FAKE, FAKE, FAKE, FAKE, 16, 100, 256, 0, FAKE, S) == SHAPE     # N % 16
    assert g(FAKE, FAKE, FAKE, FAKE, 16, 256, 256, 5, FAKE, S) == INVALID   # out dtype
    assert g(None, FAKE, FAKE, FAKE, 16, 256, 256, 0, FAKE, S) == INVALID
    assert g(FAKE, FAKE, FAKE + 1, FAKE, 16, 256, 256, 0, FAKE, S) == ALIGN
    assert g(FAKE, FAKE, FAKE, FAKE, 0, 256, 256, 0, None, S) == OK         # M == 0
    gg = F.lib.fp8_grouped_gemm
    # (qa, sa, qw, sw, off, E, total_M, N, K, out, y, stream)
    assert gg(FAKE, FAKE, FAKE, FAKE, None, 4, 16, 256, 256, 0, FAKE, S) == INVALID
    assert gg(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 16, 256, 256, 0, FAKE, S) == INVALID
    assert gg(FAKE, FAKE, FAKE, FAKE, FAKE + 2, 4, 16, 256, 256, 0, FAKE, S) == ALIGN
    assert gg(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 0, 256, 256, 0, None, S) == OK


def test_python_binding_rejects_host_tensors():
    import torch
    x = torch.zeros(4, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        F.fp8_act_quant(x, torch.zeros(4, 128, dtype=torch.uint8), torch.zeros(4, 1))


def test_python_binding_checks_gemm_operands():
    """The GEMM wrappers refuse E5M2 codes (the kernels decode E4M3) and operands
    whose shapes disagree with qa / qw, before anything reaches the library."""
    import torch
    M, N, K = 4, 256, 256
    qa = torch.zeros(M, K, dtype=torch.uint8)
    sa = torch.zeros(M, K // 128)
    qw = torch.zeros(N, K, dtype=torch.uint8)
    sw = torch.zeros(N // 128, K // 128)
    y = torch.zeros(M, N, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        F.fp8_block_gemm(qa.view(torch.float8_e5m2), sa, qw, sw, y)
    with pytest.raises(TypeError):
        F.fp8_block_gemm(qa, sa, qw.view(torch.float8_e5m2), sw, y)
    with pytest.raises(ValueError):
        F.fp8_block_gemm(qa, sa, torch.zeros(N, K + 128, dtype=torch.uint8), sw, y)   # K differs
    with pytest.raises(ValueError):
        F.fp8_block_gemm(qa, torch.zeros(M, K // 128 + 1), qw, sw, y)                 # sa shape
    with pytest.raises(ValueError):
        F.fp8_block_gemm(qa, sa, qw, torch.zeros(1, K // 128), y)                     # sw shape
    with pytest.raises(ValueError):
        F.fp8_block_gemm(qa, sa, qw, sw, torch.zeros(M, N + 16, dtype=torch.bfloat16))
    E = 3
    qwe = torch.zeros(E, N, K, dtype=torch.uint8)
    swe = torch.zeros(E, N // 128, K // 128)
    off = torch.zeros(E + 1, dtype=torch.int32)
    with pytest.raises(ValueError):
        F.fp8_grouped_gemm(qa, sa, qwe, swe, torch.zeros(E, dtype=torch.int32), y)    # offsets [E+1]
    with pytest.raises(TypeError):
        F.fp8_grouped_gemm(qa, sa, qwe, swe, off.to(torch.int64), y)
    with pytest.raises(ValueError):
        F.fp8_grouped_gemm(qa, sa, qwe, swe[:, :1].contiguous(), off, y)


def test_python_binding_refuses_stacked_weights():
    """A stacked [E, N, K] weight would be quantised as one [E*N, K] matrix whose
    128x128 blocks straddle experts; the wrapper refuses it."""
    import torch
    w = torch.zeros(2, 200, 256, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        F.fp8_weight_quant(w, torch.zeros(2, 200, 256, dtype=torch.uint8), torch.zeros(4, 2))


def test_mx_validation():
    mq = F.lib.fp8_mx_quant
    # (x, M, K, ldx, fmt, q, e8, stream)
    assert mq(FAKE, -1, 64, 64, 0, FAKE, FAKE, S) == INVALID
    assert mq(FAKE, 4, 64, 32, 0, FAKE, FAKE, S) == INVALID                # ldx < K
    assert mq(FAKE, 4, 64, 64, 3, FAKE, FAKE, S) == INVALID                # bad format
    assert mq(FAKE, 4, 72, 72, 0, FAKE, FAKE, S) == SHAPE                  # K % 16
    assert mq(FAKE, 4, 64, 64, 0, FAKE, None, S) == INVALID
    assert mq(FAKE + 8, 4, 64, 64, 0, FAKE, FAKE, S) == ALIGN
    assert mq(FAKE, 0, 64, 64, 0, None, None, S) == OK
    mg = F.lib.fp8_mx_gemm
    # (qa, sfa, qw, sfw, M, N, K, out, y, stream)
    assert mg(FAKE, FAKE, FAKE, FAKE, 16, 256, 192, 0, FAKE, S) == SHAPE    # K % 128
    assert mg(FAKE, FAKE, FAKE, FAKE, 16, 120, 256, 0, FAKE, S) == SHAPE    # N % 16
    assert mg(FAKE, FAKE, FAKE, FAKE, 16, 256, 256, 3, FAKE, S) == INVALID  # out dtype
    assert mg(FAKE, FAKE + 4, FAKE, FAKE, 16, 256, 256, 0, FAKE, S) == ALIGN  # scales: 16-byte bulk copies
    assert mg(FAKE, FAKE, FAKE, FAKE, 0, 256, 256, 0, None, S) == OK         # M == 0
    mp = F.lib.fp8_mx_pack_pow2
    # (s, rows, K, row_block, sf, stream)
    assert mp(FAKE, 16, 256, 64, FAKE, S) == INVALID                         # row block
    assert mp(FAKE, 16, 200, 1, FAKE, S) == SHAPE                            # K % 128
    assert mp(FAKE, 16, 256, 1, FAKE + 8, S) == ALIGN
    assert mp(FAKE, 0, 256, 128, None, S) == OK


def test_python_binding_checks_mx_operands():
    import torch
    M, N, K = 4, 256, 256
    qa = torch.zeros(M, K, dtype=torch.uint8)
    qw = torch.zeros(N, K, dtype=torch.uint8)
    y = torch.zeros(M, N, dtype=torch.bfloat16)
    assert F.mx_sf_bytes(M, K) == 1024 and F.mx_sf_bytes(129, 128) == 1024 and F.mx_sf_bytes(1, 16) == 512
    with pytest.raises(ValueError):      # row-major [M, K/32] bytes are not the tiled layout
        F.fp8_mx_gemm(qa, torch.zeros(M, K // 32, dtype=torch.uint8), qw,
                      torch.zeros(F.mx_sf_bytes(N, K), dtype=torch.uint8), y)
    with pytest.raises(TypeError):
        F.fp8_mx_gemm(qa, torch.zeros(F.mx_sf_bytes(M, K)), qw, torch.zeros(F.mx_sf_bytes(N, K)), y)
    with pytest.raises(ValueError):      # weight scales per 128 x 128 block
        F.fp8_mx_pack_pow2(torch.zeros(N, K // 128), N, K, 128, torch.zeros(F.mx_sf_bytes(N, K), dtype=torch.uint8))


def test_delayed_quant_validation():
    dq = F.lib.fp8_delayed_quant
    F32 = ctypes.c_float
    # (x, n, fmt, target, hist_len, algo, scale, pos, history, q, n_clipped, s_used, stream)
    assert dq(FAKE, -8, 0, F32(400.0), 16, 1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, S) == INVALID
    assert dq(FAKE, 64, 0, F32(400.0), 0, 1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, S) == INVALID    # history length
    assert dq(FAKE, 64, 0, F32(0.0), 16, 1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, S) == INVALID     # target
    assert dq(FAKE, 64, 0, F32(400.0), 16, 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, S) == INVALID   # algo
    assert dq(FAKE, 64, 5, F32(400.0), 16, 1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, S) == INVALID   # format
    assert dq(FAKE, 64, 0, F32(400.0), 16, 1, None, FAKE, FAKE, FAKE, FAKE, FAKE, S) == INVALID   # state
    assert dq(FAKE, 60, 0, F32(400.0), 16, 1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, S) == SHAPE     # n % 8
    assert dq(FAKE + 8, 64, 0, F32(400.0), 16, 1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, S) == ALIGN
    assert dq(FAKE, 64, 0, F32(400.0), 16, 1, FAKE, FAKE, FAKE, FAKE, FAKE + 4, FAKE, S) == ALIGN  # uint64 count


def test_fused_and_dequant_validation():
    gq = F.lib.fp8_block_gemm_quant
    # (qa, sa, qw, sw, M, N, K, y, fmt, scale_fmt, qy, sy, stream)
    assert gq(FAKE, FAKE, FAKE, FAKE, 16, 272, 256, None, 0, 0, FAKE, FAKE, S) == SHAPE      # N % 128
    assert gq(FAKE, FAKE, FAKE, FAKE, 16, 256, 200, None, 0, 0, FAKE, FAKE, S) == SHAPE      # K % 128
    assert gq(FAKE, FAKE, FAKE, FAKE, 16, 256, 256, None, 3, 0, FAKE, FAKE, S) == INVALID    # format
    assert gq(FAKE, FAKE, FAKE, FAKE, 16, 256, 256, None, 0, 0, FAKE, None, S) == INVALID    # sy
    assert gq(FAKE, FAKE, FAKE, FAKE, 16, 256, 256, FAKE + 2, 0, 0, FAKE, FAKE, S) == ALIGN  # y
    assert gq(FAKE, FAKE, FAKE, FAKE, 0, 256, 256, None, 0, 0, None, None, S) == OK
    dq = F.lib.fp8_weight_dequant
    # (q, s_inv, N, K, block, fmt, w, stream)
    assert dq(FAKE, FAKE, 256, 256, 64, 0, FAKE, S) == UNSUP
    assert dq(FAKE, FAKE, 256, 250, 128, 0, FAKE, S) == SHAPE
    assert dq(FAKE, FAKE, 256, 256, 128, 4, FAKE, S) == INVALID
    assert dq(FAKE, FAKE, 256, 256, 128, 0, FAKE + 8, S) == ALIGN
    assert dq(FAKE, FAKE, 0, 256, 128, 0, None, S) == OK


def test_moe_validation():
    mr = F.lib.fp8_moe_route
    # (scores, T, E, k, ids, w, offsets, row_token, row_weight, token_row, workspace, ws_bytes, stream)
    ws = F.moe_route_ws_bytes(16, 8, 1024)
    assert mr(FAKE, 16, 0, 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws, S) == INVALID       # E
    assert mr(FAKE, 16, 2048, 8, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws, S) == INVALID    # E > 1024
    assert mr(FAKE, 16, 8, 9, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws, S) == INVALID       # k > E
    assert mr(FAKE, 16, 8, 33, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws, S) == INVALID      # k > 32
    assert mr(FAKE, 16, 8, 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, ws, S) == INVALID       # no workspace
    assert mr(FAKE + 2, 16, 8, 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws, S) == ALIGN
    assert mr(FAKE, 16, 8, 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 2, ws, S) == ALIGN
    # workspace: (ceil(T*k / 512) + 1) * E int32
    assert F.moe_route_ws_bytes(4096, 8, 256) == (64 + 1) * 256 * 4
    assert mr(FAKE, 4096, 256, 8, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 65 * 256 * 4 - 4, S) == SHAPE
    mn = F.lib.fp8_moe_route_noalloc
    # (scores, T, E, k, ids, w, offsets, row_token, row_weight, token_row, stream): the
    # library's scratch holds 65536 int32; (256 + 1) * 256 of them do not fit
    assert mn(FAKE, 16384, 256, 8, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, S) == SHAPE
    assert mn(FAKE, 16, 8, 9, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, S) == INVALID
    assert mn(FAKE + 2, 16, 8, 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, S) == ALIGN
    mg = F.lib.fp8_moe_gemm
    # (qa, sa, qw, sw, offsets, row_token, row_weight, T, E, k, N, K, out, stream)
    assert mg(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16, 4, 2, 256, 200, FAKE, S) == SHAPE   # K % 128
    assert mg(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16, 4, 2, 250, 256, FAKE, S) == SHAPE   # N % 16
    assert mg(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16, 0, 2, 256, 256, FAKE, S) == INVALID
    assert mg(FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 16, 4, 2, 256, 256, FAKE, S) == INVALID
    assert mg(FAKE + 8, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16, 4, 2, 256, 256, FAKE, S) == ALIGN
    assert mg(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 4, 2, 256, 256, FAKE, S) == OK
    ap = F.lib.fp8_act_quant_permute
    # (x, T, K, ldx, fmt, scale_fmt, token_row, k, q, s, stream)
    assert ap(FAKE, 16, 256, 256, 0, 0, FAKE, 0, FAKE, FAKE, S) == INVALID      # k
    assert ap(FAKE, 16, 250, 256, 0, 0, FAKE, 2, FAKE, FAKE, S) == SHAPE        # K % 16
    assert ap(FAKE, 16, 256, 256, 0, 0, None, 2, FAKE, FAKE, S) == INVALID
    assert ap(FAKE, 16, 256, 256, 0, 0, FAKE + 2, 2, FAKE, FAKE, S) == ALIGN
    assert ap(FAKE, 0, 256, 256, 0, 0, None, 2, None, None, S) == OK


def test_header_is_plain_c_and_links(tmp_path):
    """A C99 program built against include/fp8lin.h and the library (no GPU needed)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    libdir = os.path.dirname(F.LIB_PATH)
    exe = str(tmp_path / "c_abi_check")
    cmd = [gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(root, "include"),
           "-o", exe, os.path.join(root, "tests", "c_abi_check.c"), "-L", libdir, "-lfp8lin",
           "-Wl,-rpath," + libdir]
    subprocess.run(cmd, check=True, capture_output=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and "c abi ok" in r.stdout, (r.returncode, r.stdout, r.stderr)


def test_binding_fails_loudly_without_the_library(tmp_path):
    """A copy of the binding next to no libfp8lin.so refuses to import (no fallback)."""
    import shutil
    import subprocess
    import sys
    pkg = tmp_path / "fp8_block_scaled_12_b200"
    pkg.mkdir()
    shutil.copy(os.path.join(ROOT, "fp8_block_scaled_12_b200", "__init__.py"), pkg / "__init__.py")
    r = subprocess.run([sys.executable, "-c", "import fp8_block_scaled_12_b200"], cwd=tmp_path,
                       capture_output=True, text=True, timeout=300,
                       env={**os.environ, "PYTHONPATH": str(tmp_path)})
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "libfp8lin.so is missing" in r.stderr
