"""Comparison helpers shared by the GPU parity tests (test-side only)."""
import numpy as np
import torch

import oracle as O

# Host threads for the oracle's row-parallel helpers (the oracle is plain C; the
# threads only split independent rows).
THREADS = O.default_threads()

# Every bf16 comparison records (what, elements that needed the cancellation
# allowance, elements compared); conftest prints the list at the end of the run.
ALLOWANCE_LOG = []
# At most this fraction of a comparison's elements may pass only through the
# cancellation allowance (they need |y_ref| tiny against sum |a w|).
ALLOWANCE_MAX_FRAC = 1e-3


def bits_u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def codes(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.uint8).numpy()


def assert_codes_equal(got: np.ndarray, ref: np.ndarray, what: str):
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"{what}: {len(bad)} mismatching codes, first at {bad[:5].tolist()}: " \
                          f"got {[hex(got[tuple(b)]) for b in bad[:5]]} ref {[hex(ref[tuple(b)]) for b in bad[:5]]}"


def assert_scales_equal(got: np.ndarray, ref: np.ndarray, what: str):
    g, r = got.view(np.uint32), ref.view(np.uint32)
    bad = np.argwhere(g != r)
    assert bad.size == 0, f"{what}: {len(bad)} mismatching scales, first at {bad[:5].tolist()}: " \
                          f"got {got[tuple(bad[0])]} ref {ref[tuple(bad[0])]}"


def check_fp32(y: np.ndarray, y_ref: np.ndarray, bound: np.ndarray, what: str, rel: float = 1e-5):
    """fp32 output: |y - y_ref| <= rel * sum_k |a_k w_k| per element."""
    err = np.abs(y.astype(np.float64) - y_ref)
    lim = rel * bound
    bad = np.argwhere(err > lim)
    assert bad.size == 0, f"{what}: {len(bad)} elements over tolerance; worst ratio " \
                          f"{float(np.max(err / np.maximum(lim, 1e-300))):.3g} at {bad[:3].tolist()}"
    return float(np.max(err / np.maximum(lim, 1e-300))) if err.size else 0.0


def _ord(b: np.ndarray) -> np.ndarray:
    """Monotone integer image of bf16 bit patterns (negative values mirrored)."""
    b = b.astype(np.int64)
    return np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)


def check_bf16(y_bits: np.ndarray, y_ref: np.ndarray, bound: np.ndarray, what: str, rel: float = 1e-5):
    """bf16 output: ordinal distance <= 1 from the oracle rounded straight to bf16.  An
    element may instead pass under heavy cancellation when |y - y_ref| <= rel * B plus
    half a bf16 ulp of y_ref (the fp32 accumulation error can cross more than one bf16
    ulp when |y_ref| << B).  Returns the number of elements that needed that allowance."""
    ref_bits = O.round_bf16(y_ref)
    d = np.abs(_ord(y_bits) - _ord(ref_bits))
    far = d > 1
    if far.any():
        yv = (y_bits[far].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        r = y_ref[far]
        ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(r), 2.0 ** -133))) - 7)
        ok = np.abs(yv - r) <= rel * bound[far] + 0.5 * ulp
        bad = np.argwhere(far)[~ok]
        assert bad.size == 0, f"{what}: {len(bad)} bf16 elements beyond 1 ulp and beyond the " \
                              f"cancellation allowance, first at {bad[:3].tolist()}"
    n_allow = int(far.sum())
    ALLOWANCE_LOG.append((what, n_allow, int(d.size)))
    assert n_allow <= ALLOWANCE_MAX_FRAC * d.size, \
        f"{what}: {n_allow} of {d.size} bf16 elements needed the cancellation allowance"
    return n_allow


def untile_e8m0(buf, rows: int, K: int) -> np.ndarray:
    """Tiled MXFP8 exponent bytes (the library's layout: 512-byte atoms of 128 rows x 4
    blocks, byte (r % 32) * 16 + (r % 128 / 32) * 4 + j) -> row-major [rows, ceil(K/32)],
    the oracle's layout.  A pure index permutation."""
    b = buf.detach().cpu().numpy() if isinstance(buf, torch.Tensor) else np.asarray(buf)
    nkb = (K + 127) // 128
    nb = (K + 31) // 32
    r = np.arange(rows)[:, None]
    g = np.arange(nb)[None, :]
    off = ((r >> 7) * nkb + (g >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (g & 3)
    return b[off]


def tile_e8m0(rm: np.ndarray, rows: int, K: int) -> np.ndarray:
    """Row-major [rows, K/32] exponent bytes -> the library's tiled layout (inverse of
    untile_e8m0; bytes of padding rows are 0)."""
    nkb = (K + 127) // 128
    out = np.zeros(((rows + 127) // 128) * nkb * 512, np.uint8)
    nb = rm.shape[1]
    r = np.arange(rows)[:, None]
    g = np.arange(nb)[None, :]
    off = ((r >> 7) * nkb + (g >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (g & 3)
    out[off] = rm
    return out
