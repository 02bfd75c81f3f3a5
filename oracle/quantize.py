"""Per-expert symmetric absmax quantizer.

PagedWeight, "Implementation Details", quantization scheme: for bit width b,
Q(w) = round(w / s) * s with s = max(|w|) / (2^(b-1) - 1), one scaling factor
per expert ("per-expert scaling factors").

Readings taken where the pages leave the step open:
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

import math

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


def quantization_mse(master_fp16, b: int) -> float:
    """Mean squared quantization error of one expert at b bits,
    (1/n) sum_i (w_i - Q(w_i))^2 over the expert's n fp16 weights, with the
    expert's own s and codes (quantize_expert). PagedWeight, "Quality-Aware
    Quantization", names the mean squared error as its example loss L(b) and
    ties it to the expert's sensitivity; this is that loss measured on the
    expert.

    Value: the exact sum of squares rounded once to float64, then divided by
    n in float64 (a second rounding). Exactness of the sum: w is fp16 and
    k * s is exact in float64 (8-bit k times 24-bit s), so each error
    w - k * s is an exact float64 whose bits lie at or above 2^-60 (fp16's
    smallest step is 2^-24 and s >= 2^-24 / 127 has its last bit at or above
    2^-55); scaled by 2^60 it is an integer, and the squares are summed as
    Python integers.
    """
    w = np.asarray(master_fp16)
    assert w.dtype == np.float16
    n = w.size
    if n == 0:
        return 0.0
    m, s, k = quantize_expert(w, b)
    err = w.astype(np.float64) - dequantize(k, s)
    scaled = np.ldexp(err, 60)
    assert np.array_equal(scaled, np.trunc(scaled))  # every scaled error is an integer
    total = sum(i * i for i in map(int, scaled.tolist()))
    sum_sq = math.ldexp(float(total), -120)  # float(int) rounds to nearest, ties to even
    return float(np.float64(sum_sq) / np.float64(n))
