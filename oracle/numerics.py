"""Number formats of the KV cache, written from their definitions.

TEST INFRASTRUCTURE (see ``oracle/__init__.py``).

* bfloat16: the upper 16 bits of an IEEE-754 binary32.
* FP8 E4M3 ("E4M3FN"): the OCP 8-bit floating point format. 1 sign bit, 4
  exponent bits with bias 7, 3 mantissa bits. Exponent field 0 encodes
  subnormals (-1)^s * 2^-6 * m/8. Field 15 with mantissa 7 is NaN; there is no
  infinity, so the largest finite magnitude is 2^8 * 1.75 = 448. The pages call
  this KV format "FP8" (FastDMS announcement, KV-memory table, "vLLM FP8 KV"
  column, kv_cache_dtype=fp8; the vLLM FP8-KV-by-default page enables it on
  compute-capability family 100).

Readings (the pages fix none of these):

* Quantisation of a bf16 value x with a per-head fp32 scale s:
  code = E4M3(round_to_nearest_even(fp32(x) / fp32(s))), with out-of-range
  finite quotients clamped to +-448 ("satfinite"). The quotient is the
  correctly rounded fp32 quotient; the E4M3 rounding is taken from that fp32
  value, never from a wider one (a second rounding from fp64 could differ).
* The sign of zero is kept (a negative quotient that rounds to zero gives 0x80).
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def bf16_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact fp64 values."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def bf16_to_f32(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _e4m3_value(code: int) -> float:
    """Value of one E4M3 code, straight from the field definition."""
    s = (code >> 7) & 1
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        mag = (m / 8.0) * 2.0 ** (1 - 7)
    else:
        mag = (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return -mag if s else mag


E4M3_TABLE = np.array([_e4m3_value(c) for c in range(256)], dtype=np.float64)
# non-negative finite codes 0x00..0x7E in increasing order of value
_POS_VALUES = E4M3_TABLE[:0x7F]
assert np.all(np.diff(_POS_VALUES) > 0)


def e4m3_to_f64(codes) -> np.ndarray:
    """E4M3 codes (uint8) -> exact fp64 values (NaN for 0x7F / 0xFF)."""
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_from_f32(x) -> np.ndarray:
    """fp32 values -> E4M3 codes, round to nearest (ties to even code), satfinite.

    Finite inputs only. The nearest of the two representable neighbours of |x|
    is chosen; on an exact tie the code with an even last mantissa bit wins.
    Magnitudes above 448 give 448 (0x7E / 0xFE), so NaN codes never appear.
    """
    x = np.asarray(x, dtype=np.float32)
    if not np.all(np.isfinite(x)):
        raise ValueError("e4m3_from_f32: non-finite input")
    a = np.abs(x).astype(np.float64)        # exact
    a = np.minimum(a, E4M3_MAX)
    hi = np.searchsorted(_POS_VALUES, a, side="left")   # first value >= a
    hi = np.minimum(hi, 0x7E)
    lo = np.maximum(hi - 1, 0)
    d_hi = _POS_VALUES[hi] - a
    d_lo = a - _POS_VALUES[lo]
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    sign = np.signbit(x)
    return (code | np.where(sign, 0x80, 0).astype(np.uint8)).astype(np.uint8)


def quantise_e4m3(x_bf16_bits, scale_f32, counted=None) -> tuple:
    """Quantise bf16 values with an fp32 scale: (codes uint8, saturated count).

    A value counts as saturated when |fp32(x) / scale| > 448 (it was clipped).
    ``counted``, if given, is a boolean mask over the leading axis: only those
    rows enter the count.
    """
    xf = bf16_to_f32(x_bf16_bits)
    qf = (xf / np.float32(scale_f32)).astype(np.float32)   # IEEE fp32 quotient
    clipped = np.abs(qf) > np.float32(E4M3_MAX)
    if counted is not None:
        clipped = clipped[np.asarray(counted, bool)]
    return e4m3_from_f32(qf), int(np.count_nonzero(clipped))


def calibration_scale(amax_f32) -> np.float32:
    """Per-head FP8 scale from the absolute maximum of the calibrating values.

    scale = max(amax, 2^-126) / 448, an fp32 quotient. The floor keeps the scale
    non-zero for an all-zero head.
    """
    a = np.float32(max(np.float32(amax_f32), np.float32(2.0 ** -126)))
    return np.float32(a / np.float32(E4M3_MAX))
