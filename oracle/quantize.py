"""Per-expert symmetric absmax quantizer.

PagedWeight, "Implementation Details", quantization scheme: for bit width b,
Q(w) = round(w / s) * s with s = max(|w|) / (2^(b-1) - 1), one scaling factor
per expert ("per-expert scaling factors").

Readings taken (listed in the design doc):
* max |w| runs over the whole expert (gate, up and down matrices together):
  one s per expert.
* The page calls the scheme "uniform affine" but its formula has no zero
  point: symmetric, zero point 0.
* round() is round-half-to-even of the exact real quotient w/s; the result
  is clamped to [-q_b, q_b] (a no-op safety net: |w| <= max|w|).
* s is stored as float32: s = RN_f32(m / q_b), m the exact fp16 absmax.
* m = 0 gives s = 0 and every code 0.
* NaN or Inf in the master is an error (no quantization).

Codes are stored as offset binary u = k + 2^(b-1).
"""
from __future__ import annotations

import numpy as np

from .allocate import q_levels


class NonFiniteMaster(ValueError):
    """The fp16 master holds a NaN or an infinity."""


def absmax(master_fp16) -> float:
    """m = max |w| over one expert's fp16 master, as an exact float."""
    w = np.asarray(master_fp16)
    assert w.dtype == np.float16
    if w.size == 0:
        return 0.0
    if not np.isfinite(w).all():
        raise NonFiniteMaster("master contains NaN or Inf")
    return float(np.max(np.abs(w.astype(np.float64))))


def scale(m: float, b: int) -> np.float32:
    """s = RN_f32(m / q_b): the quotient in float64, then rounded to float32."""
    return np.float32(np.float64(m) / np.float64(q_levels(b)))


def encode(w_fp16, s, b: int) -> np.ndarray:
    """k = round-half-even(w / s), clamped to [-q_b, q_b]; int64 array.

    The quotient is taken in float64. With w an fp16 value (11-bit significand)
    and s a float32 (24-bit significand), w/s is either exactly a half-integer
    or at least 2^-25 away from one, far above float64's spacing below 2^8, so
    rint of the float64 quotient equals rounding the exact quotient.
    """
    w = np.asarray(w_fp16).astype(np.float64)
    s64 = np.float64(s)
    q = q_levels(b)
    if s64 == 0.0:
        return np.zeros(w.shape, dtype=np.int64)
    k = np.rint(w / s64)
    k = np.clip(k, -q, q)
    return k.astype(np.int64)


def offset_codes(k: np.ndarray, b: int) -> np.ndarray:
    """u = k + 2^(b-1) (offset binary, 1 .. 2^b - 1)."""
    return (np.asarray(k, dtype=np.int64) + (1 << (b - 1))).astype(np.uint32)


def dequantize(k: np.ndarray, s) -> np.ndarray:
    """Q(w) = k * s in float64 (exact: 8-bit k times 24-bit s)."""
    return np.asarray(k, dtype=np.float64) * np.float64(s)


def quantize_expert(master_fp16, b: int):
    """(m, s, k) for one expert's flat fp16 master at b bits."""
    m = absmax(master_fp16)
    s = scale(m, b)
    return m, s, encode(master_fp16, s, b)
