"""B200-native FP8 W8A8 linear layer -- Python binding of libfp8lin.so.

The binding only marshals arguments: it passes device pointers, shapes and the
current CUDA stream to the C ABI declared in include/fp8lin.h, where every step
of the path runs in hand-written sm_100a kernels.  PyTorch supplies device memory
and streams.  There is no fallback: importing this package fails if the CUDA
library has not been built, and every call raises Fp8Error on a non-zero status.

Functions with the C names (``fp8_act_quant``, ``fp8_weight_quant``,
``fp8_block_gemm``, ``fp8_grouped_gemm``) take preallocated output tensors; the
short names (``act_quant``, ``weight_quant``, ``block_gemm``, ``grouped_gemm``)
allocate the outputs with torch and call them.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "E4M3", "E5M2", "SCALE_FP32", "SCALE_UE8M0", "OUT_BF16", "OUT_FP32", "Fp8Error", "LIB_PATH",
    "fp8_act_quant", "fp8_weight_quant", "fp8_block_gemm", "fp8_grouped_gemm", "fp8_mx_quant", "fp8_mx_gemm",
    "fp8_mx_pack_pow2", "fp8_delayed_quant", "DelayedScaling", "AMAX_MOST_RECENT", "AMAX_MAX",
    "fp8_block_gemm_quant", "fp8_weight_dequant", "block_gemm_quant", "weight_dequant",
    "fp8_moe_route", "fp8_moe_gemm", "fp8_act_quant_permute", "moe_route", "moe_gemm", "act_quant_permute",
    "moe_route_ws_bytes", "fp8_moe_route_noalloc", "moe_route_noalloc",
    "fp8_status_string", "fp8_device_error", "fp8_selftest_bounded_wait", "fp8_set_wait_limit_ns",
    "act_quant", "weight_quant", "block_gemm", "grouped_gemm", "mx_quant", "mx_gemm", "mx_pack_pow2",
    "mx_sf_bytes", "EXPORTS",
]

E4M3, E5M2 = 0, 1
SCALE_FP32, SCALE_UE8M0 = 0, 1
OUT_BF16, OUT_FP32 = 0, 1
MX_BLOCK = 32
AMAX_MOST_RECENT, AMAX_MAX = 0, 1
FP8_OK = 0
FP8_ERR_INVALID_SCALE = 7

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfp8lin.so")
EXPORTS = ("fp8_act_quant", "fp8_weight_quant", "fp8_block_gemm", "fp8_grouped_gemm", "fp8_mx_quant",
           "fp8_mx_gemm", "fp8_mx_pack_pow2", "fp8_delayed_quant", "fp8_block_gemm_quant", "fp8_weight_dequant",
           "fp8_moe_route", "fp8_moe_gemm", "fp8_act_quant_permute", "fp8_status_string", "fp8_device_error",
           "fp8_selftest_bounded_wait", "fp8_set_wait_limit_ns")


class Fp8Error(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {code} ({fp8_status_string(code)})")
        self.code = code


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with `python fp8_block_scaled_12_b200/build.py`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, ci = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    L.fp8_act_quant.argtypes = [vp, i64, i64, i64, ci, ci, ci, vp, vp, vp]
    L.fp8_weight_quant.argtypes = [vp, i64, i64, ci, ci, ci, vp, vp, vp]
    L.fp8_block_gemm.argtypes = [vp, vp, vp, vp, i64, i64, i64, ci, vp, vp]
    L.fp8_grouped_gemm.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, ci, vp, vp]
    L.fp8_mx_quant.argtypes = [vp, i64, i64, i64, ci, vp, vp, vp]
    L.fp8_mx_gemm.argtypes = [vp, vp, vp, vp, i64, i64, i64, ci, vp, vp]
    L.fp8_mx_pack_pow2.argtypes = [vp, i64, i64, ci, vp, vp]
    L.fp8_delayed_quant.argtypes = [vp, i64, ci, ctypes.c_float, i64, ci, vp, vp, vp, vp, vp, vp, vp]
    L.fp8_block_gemm_quant.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, ci, ci, vp, vp, vp]
    L.fp8_weight_dequant.argtypes = [vp, vp, i64, i64, ci, ci, vp, vp]
    L.fp8_moe_route.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, vp, vp, vp, i64, vp]
    L.fp8_moe_route_noalloc.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, vp, vp, vp]
    L.fp8_moe_gemm.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, vp, vp]
    L.fp8_act_quant_permute.argtypes = [vp, i64, i64, i64, ci, ci, vp, i64, vp, vp, vp]
    L.fp8_status_string.argtypes = [ci]
    L.fp8_status_string.restype = ctypes.c_char_p
    L.fp8_device_error.argtypes = [vp]
    L.fp8_selftest_bounded_wait.argtypes = [i64, vp]
    L.fp8_set_wait_limit_ns.argtypes = [i64]
    for name in ("fp8_act_quant", "fp8_weight_quant", "fp8_block_gemm", "fp8_grouped_gemm", "fp8_mx_quant",
                 "fp8_mx_gemm", "fp8_mx_pack_pow2", "fp8_delayed_quant", "fp8_block_gemm_quant",
                 "fp8_weight_dequant", "fp8_moe_route", "fp8_moe_gemm", "fp8_act_quant_permute",
                 "fp8_device_error", "fp8_selftest_bounded_wait", "fp8_set_wait_limit_ns"):
        getattr(L, name).restype = ci
    return L


lib = _load()


def fp8_status_string(code: int) -> str:
    return lib.fp8_status_string(int(code)).decode()


def _check(fn: str, code: int) -> None:
    if code != FP8_OK:
        raise Fp8Error(fn, code)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("fp8 library tensors must live on a CUDA device")
    return t.data_ptr()


def _u8(t: torch.Tensor) -> torch.Tensor:
    if t.dtype in (torch.float8_e4m3fn, torch.float8_e5m2):
        return t.view(torch.uint8)
    if t.dtype != torch.uint8:
        raise TypeError(f"FP8 codes must be uint8 / float8, got {t.dtype}")
    return t


def _e4m3_codes(t: torch.Tensor, name: str) -> torch.Tensor:
    """GEMM operands are E4M3 codes (uint8 bit patterns or float8_e4m3fn)."""
    if t.dtype == torch.float8_e5m2:
        raise TypeError(f"{name}: the GEMMs take E4M3 codes; float8_e5m2 is not supported")
    return _u8(t)


def _expect(t: torch.Tensor, shape: tuple, name: str, dtype=None) -> None:
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")


# ------------------------------------------------------------- C names
def fp8_act_quant(x: torch.Tensor, q: torch.Tensor, s: torch.Tensor, group: int = 128, fmt: int = E4M3,
                  scale_fmt: int = SCALE_FP32, stream=None) -> None:
    """Per-token, per-group quantisation of bf16 x [M, K] (row stride x.stride(0)) into
    codes q [M, K] and fp32 scales s [M, ceil(K/group)]."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    assert q.is_contiguous() and s.is_contiguous() and s.dtype == torch.float32
    M, K = x.shape
    _expect(q, (M, K), "q")
    _expect(s, (M, (K + group - 1) // group), "s")
    _check("fp8_act_quant", lib.fp8_act_quant(_ptr(x), M, K, x.stride(0), group, fmt, scale_fmt,
                                              _ptr(_u8(q)), _ptr(s), _stream(stream)))


def fp8_weight_quant(w: torch.Tensor, q: torch.Tensor, s_inv: torch.Tensor, block: int = 128,
                     fmt: int = E4M3, scale_fmt: int = SCALE_FP32, stream=None) -> None:
    """128x128-block (block=128) or per-tensor (block=0) quantisation of bf16 w [N, K]."""
    assert w.dtype == torch.bfloat16 and w.is_contiguous()
    assert q.is_contiguous() and s_inv.is_contiguous() and s_inv.dtype == torch.float32
    if w.dim() != 2:
        # a stacked [E, N, K] tensor would be quantised as one [E*N, K] matrix, whose
        # 128x128 blocks straddle experts when N % 128 != 0: quantise per expert
        raise ValueError(f"weight_quant takes one [N, K] matrix, got shape {tuple(w.shape)}; "
                         "quantise stacked expert weights one expert at a time")
    N, K = w.shape
    _expect(q, (N, K), "q")
    _expect(s_inv, (1,) if block == 0 else ((N + block - 1) // block, (K + block - 1) // block), "s_inv")
    _check("fp8_weight_quant", lib.fp8_weight_quant(_ptr(w), N, K, block, fmt, scale_fmt, _ptr(_u8(q)),
                                                    _ptr(s_inv), _stream(stream)))


def _out_code(y: torch.Tensor) -> int:
    if y.dtype == torch.bfloat16:
        return OUT_BF16
    if y.dtype == torch.float32:
        return OUT_FP32
    raise TypeError(f"output must be bf16 or fp32, got {y.dtype}")


def fp8_block_gemm(qa: torch.Tensor, sa: torch.Tensor, qw: torch.Tensor, sw: torch.Tensor, y: torch.Tensor,
                   stream=None) -> None:
    """y [M, N] = block-scaled FP8 GEMM of codes qa [M, K] (scales sa [M, K/128]) and
    qw [N, K] (scales sw [ceil(N/128), K/128])."""
    for t in (qa, sa, qw, sw, y):
        assert t.is_contiguous()
    M, K = qa.shape
    N = qw.shape[0]
    _expect(qw, (N, K), "qw")
    _expect(sa, (M, K // 128), "sa", torch.float32)
    _expect(sw, ((N + 127) // 128, K // 128), "sw", torch.float32)
    _expect(y, (M, N), "y")
    qa8, qw8, od = _e4m3_codes(qa, "qa"), _e4m3_codes(qw, "qw"), _out_code(y)
    _check("fp8_block_gemm", lib.fp8_block_gemm(_ptr(qa8), _ptr(sa), _ptr(qw8), _ptr(sw), M, N, K,
                                                od, _ptr(y), _stream(stream)))


def fp8_block_gemm_quant(qa: torch.Tensor, sa: torch.Tensor, qw: torch.Tensor, sw: torch.Tensor,
                         qy: torch.Tensor, sy: torch.Tensor, y: torch.Tensor | None = None, fmt: int = E4M3,
                         scale_fmt: int = SCALE_FP32, stream=None) -> None:
    """Block GEMM whose epilogue also quantises its bf16 output for the next layer:
    qy [M, N] codes and sy [M, N/128] scales equal act_quant(y); y (bf16 [M, N]) is
    written only when given."""
    for t in (qa, sa, qw, sw, qy, sy) + ((y,) if y is not None else ()):
        assert t.is_contiguous()
    M, K = qa.shape
    N = qw.shape[0]
    _expect(qw, (N, K), "qw")
    _expect(sa, (M, K // 128), "sa", torch.float32)
    _expect(sw, ((N + 127) // 128, K // 128), "sw", torch.float32)
    _expect(qy, (M, N), "qy")
    _expect(sy, (M, N // 128), "sy", torch.float32)
    if y is not None:
        _expect(y, (M, N), "y", torch.bfloat16)
    qa8, qw8 = _e4m3_codes(qa, "qa"), _e4m3_codes(qw, "qw")
    _check("fp8_block_gemm_quant", lib.fp8_block_gemm_quant(_ptr(qa8), _ptr(sa), _ptr(qw8), _ptr(sw), M, N, K,
                                                            _ptr(y), fmt, scale_fmt, _ptr(_u8(qy)), _ptr(sy),
                                                            _stream(stream)))


def fp8_weight_dequant(q: torch.Tensor, s_inv: torch.Tensor, w: torch.Tensor, block: int = 128,
                       fmt: int = E4M3, stream=None) -> None:
    """FP8 codes q [N, K] with scale_inv (128x128 blocks, or one scale with block=0)
    -> bf16 w [N, K]."""
    for t in (q, s_inv, w):
        assert t.is_contiguous()
    N, K = q.shape
    _expect(s_inv, (1,) if block == 0 else ((N + 127) // 128, (K + 127) // 128), "s_inv", torch.float32)
    _expect(w, (N, K), "w", torch.bfloat16)
    _check("fp8_weight_dequant", lib.fp8_weight_dequant(_ptr(_u8(q)), _ptr(s_inv), N, K, block, fmt, _ptr(w),
                                                        _stream(stream)))


def moe_route_ws_bytes(T: int, k: int, E: int) -> int:
    """Workspace of fp8_moe_route (FP8_MOE_ROUTE_WS_BYTES)."""
    return ((T * k + 511) // 512 + 1) * E * 4


def fp8_moe_route(scores: torch.Tensor, k: int, ids: torch.Tensor, w: torch.Tensor, offsets: torch.Tensor,
                  row_token: torch.Tensor, row_weight: torch.Tensor, token_row: torch.Tensor,
                  workspace: torch.Tensor, stream=None) -> None:
    """Top-k routing of fp32 scores [T, E], gate weights, and the stable expert sort
    (workspace: a device buffer of at least moe_route_ws_bytes(T, k, E) bytes)."""
    for t in (scores, ids, w, offsets, row_token, row_weight, token_row, workspace):
        assert t.is_contiguous()
    T, E = scores.shape
    _expect(scores, (T, E), "scores", torch.float32)
    _expect(ids, (T, k), "ids", torch.int32)
    _expect(w, (T, k), "w", torch.float32)
    _expect(offsets, (E + 1,), "offsets", torch.int32)
    for t, n, d in ((row_token, "row_token", torch.int32), (row_weight, "row_weight", torch.float32),
                    (token_row, "token_row", torch.int32)):
        _expect(t, (T * k,), n, d)
    nbytes = workspace.numel() * workspace.element_size()
    _check("fp8_moe_route", lib.fp8_moe_route(_ptr(scores), T, E, k, _ptr(ids), _ptr(w), _ptr(offsets),
                                              _ptr(row_token), _ptr(row_weight), _ptr(token_row), _ptr(workspace),
                                              nbytes, _stream(stream)))


def fp8_moe_route_noalloc(scores: torch.Tensor, k: int, ids: torch.Tensor, w: torch.Tensor, offsets: torch.Tensor,
                          row_token: torch.Tensor, row_weight: torch.Tensor, token_row: torch.Tensor,
                          stream=None) -> None:
    """fp8_moe_route with the library's own fixed scratch (no workspace argument)."""
    for t in (scores, ids, w, offsets, row_token, row_weight, token_row):
        assert t.is_contiguous()
    T, E = scores.shape
    _expect(scores, (T, E), "scores", torch.float32)
    _expect(ids, (T, k), "ids", torch.int32)
    _expect(w, (T, k), "w", torch.float32)
    _expect(offsets, (E + 1,), "offsets", torch.int32)
    for t, n, d in ((row_token, "row_token", torch.int32), (row_weight, "row_weight", torch.float32),
                    (token_row, "token_row", torch.int32)):
        _expect(t, (T * k,), n, d)
    _check("fp8_moe_route_noalloc", lib.fp8_moe_route_noalloc(_ptr(scores), T, E, k, _ptr(ids), _ptr(w),
                                                              _ptr(offsets), _ptr(row_token), _ptr(row_weight),
                                                              _ptr(token_row), _stream(stream)))


def fp8_act_quant_permute(x: torch.Tensor, route: dict, q: torch.Tensor, s: torch.Tensor, fmt: int = E4M3,
                          scale_fmt: int = SCALE_FP32, stream=None) -> None:
    """act_quant of bf16 x [T, K] with each token's codes / scales written to its k
    expert-sorted rows (q [T*k, K], s [T*k, ceil(K/128)])."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    T, K = x.shape
    k = route["ids"].shape[1]
    _expect(route["token_row"], (T * k,), "token_row", torch.int32)
    _expect(q, (T * k, K), "q")
    _expect(s, (T * k, (K + 127) // 128), "s", torch.float32)
    _check("fp8_act_quant_permute", lib.fp8_act_quant_permute(_ptr(x), T, K, x.stride(0), fmt, scale_fmt,
                                                              _ptr(route["token_row"]), k, _ptr(_u8(q)), _ptr(s),
                                                              _stream(stream)))


def fp8_moe_gemm(qa: torch.Tensor, sa: torch.Tensor, qw: torch.Tensor, sw: torch.Tensor, route: dict,
                 out: torch.Tensor, stream=None) -> None:
    """Expert GEMMs over the expert-sorted rows qa [T*k, K] / sa [T*k, K/128]
    (act_quant_permute) with the gate-weighted combine fused: out fp32 [T, N]."""
    for t in (qa, sa, qw, sw, out):
        assert t.is_contiguous()
    R, K = qa.shape
    E, N, _ = qw.shape
    T, k = route["ids"].shape
    _expect(qa, (T * k, K), "qa")
    _expect(qw, (E, N, K), "qw")
    _expect(sa, (T * k, K // 128), "sa", torch.float32)
    _expect(sw, (E, (N + 127) // 128, K // 128), "sw", torch.float32)
    _expect(route["offsets"], (E + 1,), "offsets", torch.int32)
    _expect(route["row_token"], (T * k,), "row_token", torch.int32)
    _expect(route["row_weight"], (T * k,), "row_weight", torch.float32)
    _expect(out, (T, N), "out", torch.float32)
    qa8, qw8 = _e4m3_codes(qa, "qa"), _e4m3_codes(qw, "qw")
    _check("fp8_moe_gemm", lib.fp8_moe_gemm(_ptr(qa8), _ptr(sa), _ptr(qw8), _ptr(sw), _ptr(route["offsets"]),
                                            _ptr(route["row_token"]), _ptr(route["row_weight"]), T, E, k, N, K,
                                            _ptr(out), _stream(stream)))


def fp8_grouped_gemm(qa: torch.Tensor, sa: torch.Tensor, qw: torch.Tensor, sw: torch.Tensor,
                     offsets: torch.Tensor, y: torch.Tensor, stream=None) -> None:
    """Grouped GEMM over expert-sorted rows: qw [E, N, K], sw [E, ceil(N/128), K/128],
    offsets device int32 [E+1]."""
    for t in (qa, sa, qw, sw, offsets, y):
        assert t.is_contiguous()
    total_M, K = qa.shape
    E, N, _ = qw.shape
    _expect(qw, (E, N, K), "qw")
    _expect(sa, (total_M, K // 128), "sa", torch.float32)
    _expect(sw, (E, (N + 127) // 128, K // 128), "sw", torch.float32)
    _expect(offsets, (E + 1,), "offsets", torch.int32)
    _expect(y, (total_M, N), "y")
    qa8, qw8, od = _e4m3_codes(qa, "qa"), _e4m3_codes(qw, "qw"), _out_code(y)
    _check("fp8_grouped_gemm", lib.fp8_grouped_gemm(_ptr(qa8), _ptr(sa), _ptr(qw8), _ptr(sw),
                                                    _ptr(offsets), E, total_M, N, K, od, _ptr(y),
                                                    _stream(stream)))


def mx_sf_bytes(rows: int, K: int) -> int:
    """Bytes of the tiled MXFP8 exponent layout of a [rows, K] operand (FP8_MX_SF_BYTES)."""
    return ((rows + 127) // 128) * ((K + 127) // 128) * 512


def fp8_mx_quant(x: torch.Tensor, q: torch.Tensor, e8: torch.Tensor, fmt: int = E4M3, stream=None) -> None:
    """MXFP8 quantisation of bf16 x [M, K] (row stride x.stride(0)) into codes q [M, K]
    and E8M0 exponent bytes e8 (uint8, mx_sf_bytes(M, K), tiled layout of the header)."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    assert q.is_contiguous() and e8.is_contiguous()
    M, K = x.shape
    _expect(q, (M, K), "q")
    _expect(e8, (mx_sf_bytes(M, K),), "e8", torch.uint8)
    _check("fp8_mx_quant", lib.fp8_mx_quant(_ptr(x), M, K, x.stride(0), fmt, _ptr(_u8(q)), _ptr(e8),
                                            _stream(stream)))


def fp8_mx_gemm(qa: torch.Tensor, sfa: torch.Tensor, qw: torch.Tensor, sfw: torch.Tensor, y: torch.Tensor,
                stream=None) -> None:
    """y [M, N] = FP8 GEMM with E8M0 scales per 32-element block of K applied by the
    tensor core; sfa / sfw are tiled exponent bytes (mx_quant, or mx_pack_pow2 for the
    ue8m0 scales of act_quant / weight_quant)."""
    for t in (qa, sfa, qw, sfw, y):
        assert t.is_contiguous()
    M, K = qa.shape
    N = qw.shape[0]
    _expect(qw, (N, K), "qw")
    _expect(sfa, (mx_sf_bytes(M, K),), "sfa", torch.uint8)
    _expect(sfw, (mx_sf_bytes(N, K),), "sfw", torch.uint8)
    _expect(y, (M, N), "y")
    qa8, qw8, od = _e4m3_codes(qa, "qa"), _e4m3_codes(qw, "qw"), _out_code(y)
    _check("fp8_mx_gemm", lib.fp8_mx_gemm(_ptr(qa8), _ptr(sfa), _ptr(qw8), _ptr(sfw), M, N, K, od, _ptr(y),
                                          _stream(stream)))


def fp8_mx_pack_pow2(s: torch.Tensor, rows: int, K: int, row_block: int, sf: torch.Tensor, stream=None) -> None:
    """fp32 power-of-two scales in the block GEMM's layout (row_block 1: [rows, K/128];
    128: [ceil(rows/128), K/128]) -> tiled exponent bytes sf (mx_sf_bytes(rows, K))."""
    assert s.dtype == torch.float32 and s.is_contiguous() and sf.is_contiguous()
    _expect(s, (rows if row_block == 1 else (rows + 127) // 128, K // 128), "s")
    _expect(sf, (mx_sf_bytes(rows, K),), "sf", torch.uint8)
    _check("fp8_mx_pack_pow2", lib.fp8_mx_pack_pow2(_ptr(s), rows, K, row_block, _ptr(sf), _stream(stream)))


def fp8_delayed_quant(x: torch.Tensor, q: torch.Tensor, scale: torch.Tensor, pos: torch.Tensor,
                      history: torch.Tensor, n_clipped: torch.Tensor, s_used: torch.Tensor, fmt: int = E4M3,
                      target: float = 400.0, algo: int = AMAX_MAX, stream=None) -> None:
    """One delayed-scaling step over all elements of bf16 x (any shape, contiguous)."""
    for t in (x, q, scale, pos, history, n_clipped, s_used):
        assert t.is_contiguous()
    assert x.dtype == torch.bfloat16 and q.numel() == x.numel()
    _expect(scale, (1,), "scale", torch.float32)
    _expect(pos, (1,), "pos", torch.int32)
    assert history.dtype == torch.float32 and history.dim() == 1
    _expect(n_clipped, (1,), "n_clipped", torch.int64)
    _expect(s_used, (1,), "s_used", torch.float32)
    _check("fp8_delayed_quant", lib.fp8_delayed_quant(_ptr(x), x.numel(), fmt, float(target), history.numel(),
                                                      algo, _ptr(scale), _ptr(pos), _ptr(history), _ptr(_u8(q)),
                                                      _ptr(n_clipped), _ptr(s_used), _stream(stream)))


class DelayedScaling:
    """Device state of delayed per-tensor scaling (initial scale 1.0, empty history),
    stepped with fp8_delayed_quant; `step(x)` returns (codes, scale used, clipped count
    as a device tensor)."""

    def __init__(self, hist_len: int = 16, fmt: int = E4M3, target: float | None = None,
                 algo: int = AMAX_MAX, device="cuda"):
        self.fmt, self.algo = fmt, algo
        self.target = target if target is not None else (400.0 if fmt == E4M3 else 57344.0 * 400.0 / 448.0)
        self.scale = torch.ones(1, dtype=torch.float32, device=device)
        self.pos = torch.zeros(1, dtype=torch.int32, device=device)
        self.history = torch.zeros(hist_len, dtype=torch.float32, device=device)

    def step(self, x: torch.Tensor, stream=None):
        q = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
        n_clipped = torch.empty(1, dtype=torch.int64, device=x.device)
        s_used = torch.empty(1, dtype=torch.float32, device=x.device)
        fp8_delayed_quant(x, q, self.scale, self.pos, self.history, n_clipped, s_used, self.fmt, self.target,
                          self.algo, stream)
        return q, s_used, n_clipped


def fp8_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device-side wait status."""
    return int(lib.fp8_device_error(_stream(stream)))


def fp8_selftest_bounded_wait(limit_ns: int, stream=None) -> None:
    """Launch the diagnostic kernel whose bounded mbarrier wait runs out after
    `limit_ns`; a following fp8_device_error() reports the timeout."""
    _check("fp8_selftest_bounded_wait", lib.fp8_selftest_bounded_wait(int(limit_ns), _stream(stream)))


def fp8_set_wait_limit_ns(limit_ns: int) -> None:
    """Diagnostic: limit of the GEMM kernels' bounded waits (0 restores the default)."""
    _check("fp8_set_wait_limit_ns", lib.fp8_set_wait_limit_ns(int(limit_ns)))


# ------------------------------------------------- allocating wrappers
def act_quant(x: torch.Tensor, group: int = 128, fmt: int = E4M3, scale_fmt: int = SCALE_FP32, stream=None):
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    s = torch.empty((M, (K + group - 1) // group), dtype=torch.float32, device=x.device)
    fp8_act_quant(x, q, s, group, fmt, scale_fmt, stream)
    return q, s


def weight_quant(w: torch.Tensor, block: int = 128, fmt: int = E4M3, scale_fmt: int = SCALE_FP32,
                 stream=None):
    N, K = w.shape
    q = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    shape = (1,) if block == 0 else ((N + block - 1) // block, (K + block - 1) // block)
    s = torch.empty(shape, dtype=torch.float32, device=w.device)
    fp8_weight_quant(w, q, s, block, fmt, scale_fmt, stream)
    return q, s


def block_gemm(qa, sa, qw, sw, out_dtype=torch.bfloat16, stream=None):
    y = torch.empty((qa.shape[0], qw.shape[0]), dtype=out_dtype, device=qa.device)
    fp8_block_gemm(qa, sa, qw, sw, y, stream)
    return y


def grouped_gemm(qa, sa, qw, sw, offsets, out_dtype=torch.bfloat16, stream=None):
    y = torch.empty((qa.shape[0], qw.shape[1]), dtype=out_dtype, device=qa.device)
    fp8_grouped_gemm(qa, sa, qw, sw, offsets, y, stream)
    return y


def mx_quant(x: torch.Tensor, fmt: int = E4M3, stream=None):
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    e8 = torch.empty((mx_sf_bytes(M, K),), dtype=torch.uint8, device=x.device)
    fp8_mx_quant(x, q, e8, fmt, stream)
    return q, e8


def mx_gemm(qa, sfa, qw, sfw, out_dtype=torch.bfloat16, stream=None):
    y = torch.empty((qa.shape[0], qw.shape[0]), dtype=out_dtype, device=qa.device)
    fp8_mx_gemm(qa, sfa, qw, sfw, y, stream)
    return y


def mx_pack_pow2(s: torch.Tensor, rows: int, K: int, row_block: int, stream=None):
    sf = torch.empty((mx_sf_bytes(rows, K),), dtype=torch.uint8, device=s.device)
    fp8_mx_pack_pow2(s, rows, K, row_block, sf, stream)
    return sf


def block_gemm_quant(qa, sa, qw, sw, fmt: int = E4M3, scale_fmt: int = SCALE_FP32, with_y: bool = False,
                     stream=None):
    M, N = qa.shape[0], qw.shape[0]
    qy = torch.empty((M, N), dtype=torch.uint8, device=qa.device)
    sy = torch.empty((M, N // 128), dtype=torch.float32, device=qa.device)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=qa.device) if with_y else None
    fp8_block_gemm_quant(qa, sa, qw, sw, qy, sy, y, fmt, scale_fmt, stream)
    return (qy, sy, y) if with_y else (qy, sy)


def weight_dequant(q, s_inv, block: int = 128, fmt: int = E4M3, stream=None):
    w = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    fp8_weight_dequant(q, s_inv, w, block, fmt, stream)
    return w


def moe_route(scores: torch.Tensor, k: int, stream=None) -> dict:
    T, E = scores.shape
    dev = scores.device
    r = dict(ids=torch.empty((T, k), dtype=torch.int32, device=dev),
             w=torch.empty((T, k), dtype=torch.float32, device=dev),
             offsets=torch.empty((E + 1,), dtype=torch.int32, device=dev),
             row_token=torch.empty((T * k,), dtype=torch.int32, device=dev),
             row_weight=torch.empty((T * k,), dtype=torch.float32, device=dev),
             token_row=torch.empty((T * k,), dtype=torch.int32, device=dev),
             workspace=torch.empty((moe_route_ws_bytes(T, k, E) // 4,), dtype=torch.int32, device=dev))
    fp8_moe_route(scores, k, r["ids"], r["w"], r["offsets"], r["row_token"], r["row_weight"], r["token_row"],
                  r["workspace"], stream)
    return r


def moe_route_noalloc(scores: torch.Tensor, k: int, stream=None) -> dict:
    T, E = scores.shape
    dev = scores.device
    r = dict(ids=torch.empty((T, k), dtype=torch.int32, device=dev),
             w=torch.empty((T, k), dtype=torch.float32, device=dev),
             offsets=torch.empty((E + 1,), dtype=torch.int32, device=dev),
             row_token=torch.empty((T * k,), dtype=torch.int32, device=dev),
             row_weight=torch.empty((T * k,), dtype=torch.float32, device=dev),
             token_row=torch.empty((T * k,), dtype=torch.int32, device=dev))
    fp8_moe_route_noalloc(scores, k, r["ids"], r["w"], r["offsets"], r["row_token"], r["row_weight"], r["token_row"],
                          stream)
    return r


def act_quant_permute(x: torch.Tensor, route: dict, fmt: int = E4M3, scale_fmt: int = SCALE_FP32, stream=None):
    T, K = x.shape
    k = route["ids"].shape[1]
    q = torch.empty((T * k, K), dtype=torch.uint8, device=x.device)
    s = torch.empty((T * k, (K + 127) // 128), dtype=torch.float32, device=x.device)
    fp8_act_quant_permute(x, route, q, s, fmt, scale_fmt, stream)
    return q, s


def moe_gemm(qa, sa, qw, sw, route: dict, stream=None):
    out = torch.empty((route["ids"].shape[0], qw.shape[1]), dtype=torch.float32, device=qa.device)
    fp8_moe_gemm(qa, sa, qw, sw, route, out, stream)
    return out
