"""CPU oracle for the FP8 W8A8 linear layer -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline / reference leg
of ``bench.py`` may import this package.  The product library never does, and
the oracle shares no code with it: the arithmetic lives in ``fp8_oracle.c``
(plain C, scalar loops, fp64 GEMM) and this module only marshals numpy arrays.

Every function cites the passage it follows in ``fp8_oracle.c``.  Parity is
pinned by ``tests/test_oracle_*.py`` against values the pages fix (E4M3 max 448,
E5M2 max 57344), closed forms, library casts and hand-computed cases.
"""
from __future__ import annotations

import ctypes
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from . import build as _build

E4M3, E5M2 = 0, 1
SCALE_FP32, SCALE_UE8M0 = 0, 1

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        L.orc_decode.restype = ctypes.c_double
        L.orc_decode.argtypes = [ctypes.c_uint8, ctypes.c_int]
        L.orc_encode.restype = ctypes.c_uint8
        L.orc_encode.argtypes = [ctypes.c_float, ctypes.c_int]
        L.orc_fmax.restype = ctypes.c_double
        L.orc_fmax.argtypes = [ctypes.c_int]
        L.orc_scale_from_amax.restype = ctypes.c_float
        L.orc_scale_from_amax.argtypes = [ctypes.c_float, ctypes.c_int, ctypes.c_int]
        L.orc_round_bf16.restype = ctypes.c_uint16
        L.orc_round_bf16.argtypes = [ctypes.c_double]
        vp = ctypes.c_void_p
        i64 = ctypes.c_int64
        L.orc_act_quant.restype = None
        L.orc_act_quant.argtypes = [vp, i64, i64, i64, i64, ctypes.c_int, ctypes.c_int, vp, vp]
        L.orc_weight_quant_block.restype = None
        L.orc_weight_quant_block.argtypes = [vp, i64, i64, i64, ctypes.c_int, ctypes.c_int, vp, vp]
        L.orc_cast_with_scale.restype = None
        L.orc_cast_with_scale.argtypes = [vp, i64, ctypes.c_float, ctypes.c_int, vp]
        L.orc_tensor_quant.restype = None
        L.orc_tensor_quant.argtypes = [vp, i64, ctypes.c_int, ctypes.c_int, vp, vp]
        L.orc_gemm_rows.restype = None
        L.orc_gemm_rows.argtypes = [vp, vp, vp, vp, i64, i64, vp, i64, vp, vp]
        L.orc_e8m0_decode.restype = ctypes.c_double
        L.orc_e8m0_decode.argtypes = [ctypes.c_uint8]
        L.orc_mx_quant.restype = None
        L.orc_mx_quant.argtypes = [vp, i64, i64, i64, i64, ctypes.c_int, vp, vp]
        L.orc_mx_gemm_rows.restype = None
        L.orc_mx_gemm_rows.argtypes = [vp, vp, vp, vp, i64, i64, vp, i64, vp, vp]
        L.orc_moe_route.restype = None
        L.orc_moe_route.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, vp, vp]
        L.orc_moe_combine_rows.restype = None
        L.orc_moe_combine_rows.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp, i64, vp, vp]
        L.orc_weight_dequant.restype = None
        L.orc_weight_dequant.argtypes = [vp, vp, i64, i64, i64, ctypes.c_int, vp]
        L.orc_delayed_quant.restype = None
        L.orc_delayed_quant.argtypes = [vp, i64, ctypes.c_int, ctypes.c_float, i64, ctypes.c_int, vp, vp, vp, vp,
                                        vp, vp]
        L.orc_grouped_gemm_rows.restype = None
        L.orc_grouped_gemm_rows.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, vp, i64, vp, vp]
        del u8p
        _lib = L
    return _lib


def default_threads() -> int:
    """Host threads the row-parallel helpers use: every core this process may run on."""
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def _split(n: int, parts: int, align: int = 1):
    """[start, stop) ranges covering [0, n) in at most `parts` pieces, boundaries on multiples of align."""
    units = (n + align - 1) // align
    parts = max(1, min(parts, units))
    bounds = [min(n, (units * i // parts) * align) for i in range(parts + 1)]
    return [(a, b) for a, b in zip(bounds[:-1], bounds[1:]) if b > a]


def _run_parallel(fn, ranges, threads: int):
    """Run fn(start, stop) over the ranges on `threads` host threads (the C calls
    release the GIL), in order of the ranges."""
    if threads <= 1 or len(ranges) <= 1:
        return [fn(a, b) for a, b in ranges]
    with ThreadPoolExecutor(max_workers=threads) as ex:
        return list(ex.map(lambda r: fn(*r), ranges))


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _bf16_bits(x) -> np.ndarray:
    """Accept a uint16 array of bf16 bit patterns or a torch bf16 CPU tensor."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch
    assert x.dtype == torch.bfloat16 and x.device.type == "cpu"
    return np.ascontiguousarray(x.contiguous().view(torch.int16).numpy().view(np.uint16))


# ----------------------------------------------------------------- codec
def decode(code: int, fmt: int = E4M3) -> float:
    return lib().orc_decode(code & 0xFF, fmt)


def encode(x: float, fmt: int = E4M3) -> int:
    return int(lib().orc_encode(x, fmt))


def fmax(fmt: int = E4M3) -> float:
    return lib().orc_fmax(fmt)


def scale_from_amax(amax: float, fmt: int = E4M3, scale_fmt: int = SCALE_FP32) -> float:
    return float(lib().orc_scale_from_amax(amax, fmt, scale_fmt))


def decode_table(fmt: int = E4M3) -> np.ndarray:
    """fp64 value of each of the 256 codes (NaN where the code is NaN)."""
    return np.array([decode(c, fmt) for c in range(256)], dtype=np.float64)


def round_bf16(v: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 bit patterns, one direct round-to-nearest-even."""
    f = lib().orc_round_bf16
    flat = np.asarray(v, dtype=np.float64).ravel()
    out = np.fromiter((f(float(t)) for t in flat), dtype=np.uint16, count=flat.size)
    return out.reshape(np.shape(v))


# ------------------------------------------------------------ quantisers
def act_quant(x, group: int = 128, fmt: int = E4M3, scale_fmt: int = SCALE_FP32, threads: int = 1):
    """x: [M, K] bf16 (bits or torch tensor) -> (q uint8 [M, K], s fp32 [M, ceil(K/group)]).
    threads > 1 splits the rows (independent) over host threads."""
    xb = _bf16_bits(x)
    M, K = xb.shape
    ng = (K + group - 1) // group
    q = np.empty((M, K), dtype=np.uint8)
    s = np.empty((M, ng), dtype=np.float32)

    def part(r0, r1):
        lib().orc_act_quant(_ptr(xb) + r0 * K * 2, r1 - r0, K, K, group, fmt, scale_fmt,
                            _ptr(q) + r0 * K, _ptr(s) + r0 * ng * 4)

    _run_parallel(part, _split(M, threads), threads)
    return q, s


def weight_quant(w, block: int = 128, fmt: int = E4M3, scale_fmt: int = SCALE_FP32, threads: int = 1):
    """w: [N, K] bf16 -> (q uint8 [N, K], s_inv fp32 [ceil(N/b), ceil(K/b)]); block=0 is per-tensor.
    threads > 1 splits the block rows (independent) over host threads."""
    wb = _bf16_bits(w)
    N, K = wb.shape
    q = np.empty((N, K), dtype=np.uint8)
    if block == 0:
        s = np.empty((1,), dtype=np.float32)
        lib().orc_tensor_quant(_ptr(wb), N * K, fmt, scale_fmt, _ptr(q), _ptr(s))
        return q, s
    nbk = (K + block - 1) // block
    s = np.empty(((N + block - 1) // block, nbk), dtype=np.float32)

    def part(r0, r1):
        lib().orc_weight_quant_block(_ptr(wb) + r0 * K * 2, r1 - r0, K, block, fmt, scale_fmt,
                                     _ptr(q) + r0 * K, _ptr(s) + (r0 // block) * nbk * 4)

    _run_parallel(part, _split(N, threads, block), threads)
    return q, s


def tensor_quant(x, fmt: int = E4M3, scale_fmt: int = SCALE_FP32):
    """Per-tensor quantisation of any bf16 array -> (q uint8 same shape, s fp32 [1])."""
    xb = _bf16_bits(x)
    q = np.empty(xb.shape, dtype=np.uint8)
    s = np.empty((1,), dtype=np.float32)
    lib().orc_tensor_quant(_ptr(xb), xb.size, fmt, scale_fmt, _ptr(q), _ptr(s))
    return q, s


def cast_with_scale(x, s: float, fmt: int = E4M3):
    """Codes of bf16 x under a given scale: FP8Cast(x / s), same shape as x."""
    xb = _bf16_bits(x)
    q = np.empty(xb.shape, dtype=np.uint8)
    lib().orc_cast_with_scale(_ptr(xb), xb.size, float(s), fmt, _ptr(q))
    return q


# ------------------------------------------------------------------ GEMM
def gemm_rows(qa, sa, qw, sw, rows=None, threads: int = 1):
    """fp64 block-scaled GEMM on the given rows -> (y [nr, N] fp64, bound [nr, N] fp64).
    threads > 1 splits the rows over host threads."""
    qa = np.ascontiguousarray(qa, dtype=np.uint8)
    qw = np.ascontiguousarray(qw, dtype=np.uint8)
    sa = np.ascontiguousarray(sa, dtype=np.float32)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    M, K = qa.shape
    N = qw.shape[0]
    assert K % 128 == 0 and qw.shape[1] == K
    rows = np.arange(M, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    y = np.empty((rows.size, N), dtype=np.float64)
    b = np.empty((rows.size, N), dtype=np.float64)

    def part(i0, i1):
        lib().orc_gemm_rows(_ptr(qa), _ptr(sa), _ptr(qw), _ptr(sw), N, K, _ptr(rows) + i0 * 8, i1 - i0,
                            _ptr(y) + i0 * N * 8, _ptr(b) + i0 * N * 8)

    _run_parallel(part, _split(rows.size, threads), threads)
    return y, b


def grouped_gemm_rows(qa, sa, qw, sw, offsets, rows, threads: int = 1):
    """Grouped GEMM on selected rows.  qw: [E, N, K], sw: [E, ceil(N/128), K/128], offsets int32 [E+1].
    threads > 1 splits the rows over host threads."""
    qa = np.ascontiguousarray(qa, dtype=np.uint8)
    qw = np.ascontiguousarray(qw, dtype=np.uint8)
    sa = np.ascontiguousarray(sa, dtype=np.float32)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    off = np.ascontiguousarray(offsets, dtype=np.int32)
    E, N, K = qw.shape
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    y = np.empty((rows.size, N), dtype=np.float64)
    b = np.empty((rows.size, N), dtype=np.float64)

    def part(i0, i1):
        lib().orc_grouped_gemm_rows(_ptr(qa), _ptr(sa), _ptr(qw), _ptr(sw), _ptr(off), E, N, K,
                                    _ptr(rows) + i0 * 8, i1 - i0, _ptr(y) + i0 * N * 8, _ptr(b) + i0 * N * 8)

    _run_parallel(part, _split(rows.size, threads), threads)
    return y, b


# ----------------------------------------------------------------- MXFP8
MX_BLOCK = 32


def e8m0_decode(b: int) -> float:
    """Value 2^(b-127) of an E8M0 shared-exponent byte (0xFF is NaN)."""
    return lib().orc_e8m0_decode(b & 0xFF)


def mx_quant(x, fmt: int = E4M3, block: int = MX_BLOCK, threads: int = 1):
    """MXFP8: x [M, K] bf16 -> (q uint8 [M, K], e8 uint8 [M, ceil(K/block)]) with one E8M0
    exponent per `block` consecutive elements of a row."""
    xb = _bf16_bits(x)
    M, K = xb.shape
    nb = (K + block - 1) // block
    q = np.empty((M, K), dtype=np.uint8)
    e8 = np.empty((M, nb), dtype=np.uint8)

    def part(r0, r1):
        lib().orc_mx_quant(_ptr(xb) + r0 * K * 2, r1 - r0, K, K, block, fmt, _ptr(q) + r0 * K,
                           _ptr(e8) + r0 * nb)

    _run_parallel(part, _split(M, threads), threads)
    return q, e8


def mx_gemm_rows(qa, ea, qw, ew, rows=None, threads: int = 1):
    """fp64 MXFP8 GEMM on the given rows (32-element E8M0 blocks along K on both
    operands) -> (y [nr, N], bound [nr, N])."""
    qa = np.ascontiguousarray(qa, dtype=np.uint8)
    qw = np.ascontiguousarray(qw, dtype=np.uint8)
    ea = np.ascontiguousarray(ea, dtype=np.uint8)
    ew = np.ascontiguousarray(ew, dtype=np.uint8)
    M, K = qa.shape
    N = qw.shape[0]
    assert K % MX_BLOCK == 0 and qw.shape[1] == K
    assert ea.shape == (M, K // MX_BLOCK) and ew.shape == (N, K // MX_BLOCK)
    rows = np.arange(M, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    y = np.empty((rows.size, N), dtype=np.float64)
    b = np.empty((rows.size, N), dtype=np.float64)

    def part(i0, i1):
        lib().orc_mx_gemm_rows(_ptr(qa), _ptr(ea), _ptr(qw), _ptr(ew), N, K, _ptr(rows) + i0 * 8, i1 - i0,
                               _ptr(y) + i0 * N * 8, _ptr(b) + i0 * N * 8)

    _run_parallel(part, _split(rows.size, threads), threads)
    return y, b


# ------------------------------------------------------- delayed scaling
ALGO_MOST_RECENT, ALGO_MAX = 0, 1


class DelayedScalingState:
    """Host copy of the delayed-scaling state: the scale for the next step (starts at
    1.0), the history ring of past amaxes and the slot the next amax goes to."""

    def __init__(self, hist_len: int = 16):
        self.scale = np.array([1.0], np.float32)
        self.pos = np.array([0], np.int32)
        self.history = np.zeros(hist_len, np.float32)


def delayed_quant(x, state: DelayedScalingState, fmt: int = E4M3, target: float = 400.0, algo: int = ALGO_MAX):
    """One step: codes of x under the previous step's scale, the number of clipped
    elements, the scale used; `state` is updated in place for the next step."""
    xb = _bf16_bits(x)
    q = np.empty(xb.shape, dtype=np.uint8)
    n_clip = np.zeros(1, np.uint64)
    s_used = np.zeros(1, np.float32)
    lib().orc_delayed_quant(_ptr(xb), xb.size, fmt, float(target), state.history.size, algo, _ptr(state.scale),
                            _ptr(state.pos), _ptr(state.history), _ptr(q), _ptr(n_clip), _ptr(s_used))
    return q, int(n_clip[0]), float(s_used[0])


def weight_dequant(q, s_inv, block: int = 128, fmt: int = E4M3, threads: int = 1):
    """FP8 codes [N, K] + scales -> bf16 bit patterns [N, K] (fp32 product, one RNE to bf16)."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    s_inv = np.ascontiguousarray(s_inv, dtype=np.float32)
    N, K = q.shape
    out = np.empty((N, K), dtype=np.uint16)
    nbk = (K + block - 1) // block if block else 1

    def part(r0, r1):
        sp = _ptr(s_inv) + ((r0 // block) * nbk * 4 if block else 0)
        lib().orc_weight_dequant(_ptr(q) + r0 * K, sp, r1 - r0, K, block, fmt, _ptr(out) + r0 * K * 2)

    _run_parallel(part, _split(N, threads, block if block else 1), threads)
    return out


# ------------------------------------------------------------ MoE routing
def moe_route(scores, k: int):
    """scores fp32 [T, E] -> dict(ids, w [T, k], offsets [E+1], row_token, row_weight,
    token_row [T*k])."""
    sc = np.ascontiguousarray(scores, dtype=np.float32)
    T, E = sc.shape
    r = dict(ids=np.empty((T, k), np.int32), w=np.empty((T, k), np.float32), offsets=np.empty(E + 1, np.int32),
             row_token=np.empty(T * k, np.int32), row_weight=np.empty(T * k, np.float32),
             token_row=np.empty(T * k, np.int32))
    lib().orc_moe_route(_ptr(sc), T, E, k, _ptr(r["ids"]), _ptr(r["w"]), _ptr(r["offsets"]), _ptr(r["row_token"]),
                        _ptr(r["row_weight"]), _ptr(r["token_row"]))
    return r


def moe_combine_rows(qa, sa, qw, sw, ids, w, tokens, threads: int = 1):
    """fp64 MoE output rows out[t] = sum_j w[t][j] * GEMM(qa[t], expert ids[t][j]) for the
    listed tokens -> (out [nt, N], bound [nt, N])."""
    qa = np.ascontiguousarray(qa, dtype=np.uint8)
    sa = np.ascontiguousarray(sa, dtype=np.float32)
    qw = np.ascontiguousarray(qw, dtype=np.uint8)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    E, N, K = qw.shape
    k = ids.shape[1]
    tokens = np.ascontiguousarray(tokens, dtype=np.int64)
    out = np.empty((tokens.size, N), np.float64)
    bound = np.empty((tokens.size, N), np.float64)

    def part(i0, i1):
        lib().orc_moe_combine_rows(_ptr(qa), _ptr(sa), _ptr(qw), _ptr(sw), _ptr(ids), _ptr(w), k, N, K,
                                   _ptr(tokens) + i0 * 8, i1 - i0, _ptr(out) + i0 * N * 8, _ptr(bound) + i0 * N * 8)

    _run_parallel(part, _split(tokens.size, threads), threads)
    return out, bound
