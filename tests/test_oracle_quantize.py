"""Pins for oracle.quantize (PagedWeight, "Implementation Details", quantization
scheme: Q(w) = round(w/s) s, s = max|w| / (2^(b-1) - 1)).

Pins: a hand-worked example at each width, exact rational rounding
(fractions.Fraction) over exhaustive fp16 sweeps, the scale's single rounding
to float32 checked exactly, and the invariants the formula fixes:
|Q(w) - w| <= s/2, |k| <= q_b, the largest-magnitude weight maps to +-q_b s,
and Q(Q(w)) = Q(w).
"""
from fractions import Fraction

import numpy as np
import pytest

from oracle import quantize as Qz
from oracle.allocate import q_levels


def rne_fraction(x: Fraction) -> int:
    """Round a rational to the nearest integer, ties to even (Python's round)."""
    return round(x)


def rn_f32(x: Fraction) -> np.float32:
    """Round a rational to the nearest float32, ties to even, by exact comparison."""
    c = np.float32(float(x))
    cands = [np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))]
    best = None
    for f in cands:
        d = abs(Fraction(float(f)) - x)
        key = (d, int(np.frombuffer(np.float32(f).tobytes(), np.uint32)[0]) & 1)
        if best is None or key < best[0]:
            best = (key, f)
    return np.float32(best[1])


# Worked by hand from the formula (round half to even):
#  b=3: max|w| = 1.5, q = 3 -> s = 0.5; w/s = 3, -1.5, 0.5, 1, -2, 0.25
#  b=4: max|w| = 0.875, q = 7 -> s = 0.125; w/s = 7, -2.5, 0.5, -1.5, 4, -3.5
#  b=8: max|w| = 127/128, q = 127 -> s = 2^-7; w/s = 127, -0.5, 1.5, -64, 38.40625
#       (0.300048828125 is fp16(0.3))
HAND = [
    (3, [1.5, -0.75, 0.25, 0.5, -1.0, 0.125], 0.5, [3, -2, 0, 1, -2, 0],
     [1.5, -1.0, 0.0, 0.5, -1.0, 0.0]),
    (4, [0.875, -0.3125, 0.0625, -0.1875, 0.5, -0.4375], 0.125, [7, -2, 0, -2, 4, -4],
     [0.875, -0.25, 0.0, -0.25, 0.5, -0.5]),
    (8, [0.9921875, -0.00390625, 0.01171875, -0.5, 0.300048828125], 0.0078125,
     [127, 0, 2, -64, 38], [0.9921875, 0.0, 0.015625, -0.5, 0.296875]),
]


@pytest.mark.parametrize("b,w,s,k,q", HAND)
def test_hand_worked_example(b, w, s, k, q):
    w16 = np.array(w, dtype=np.float16)
    assert list(w16.astype(np.float64)) == w  # inputs are exact fp16 values
    m, s_, k_ = Qz.quantize_expert(w16, b)
    assert m == max(abs(x) for x in w)
    assert float(s_) == s
    assert list(k_) == k
    assert list(Qz.dequantize(k_, s_)) == q


def all_finite_fp16():
    bits = np.arange(0, 0x10000, dtype=np.uint32).astype(np.uint16)
    v = bits.view(np.float16)
    return v[np.isfinite(v)]


def test_scale_is_single_rounding_exhaustive():
    # for every positive finite fp16 m and q in {3,7,127}: float32(float64(m)/q)
    # equals the float32 nearest to the exact rational m/q
    pos = all_finite_fp16()
    pos = np.unique(pos[pos > 0].astype(np.float64))
    for b in (3, 4, 8):
        q = q_levels(b)
        got = np.array([Qz.scale(m, b) for m in pos], dtype=np.float32)
        for i in range(0, len(pos), 97):   # exact check on a stride through all values
            assert got[i] == rn_f32(Fraction(pos[i]) / q)
        # and every value: no float64 quotient lies on a float32 midpoint
        quot = pos / q
        f32 = quot.astype(np.float32).astype(np.float64)
        lo = np.nextafter(quot.astype(np.float32), np.float32(-np.inf)).astype(np.float64)
        hi = np.nextafter(quot.astype(np.float32), np.float32(np.inf)).astype(np.float64)
        assert not np.any(quot == (f32 + lo) / 2)
        assert not np.any(quot == (f32 + hi) / 2)


@pytest.mark.parametrize("b", [3, 4, 8])
@pytest.mark.parametrize("m", [0.199951171875, 0.0935668945, 1.0, 6.103515625e-05, 65504.0])
def test_encode_exact_rational_sweep(b, m):
    # every finite fp16 w with |w| <= m: float64 rint == exact round-half-even
    m = float(np.float16(m))
    allv = all_finite_fp16()
    w = allv[np.abs(allv.astype(np.float64)) <= m]
    s = Qz.scale(m, b)
    k = Qz.encode(w, s, b)
    S = Fraction(float(s))
    q = q_levels(b)
    stride = 1 if len(w) < 20000 else 7
    for i in range(0, len(w), stride):
        exact = rne_fraction(Fraction(float(w[i])) / S)
        exact = max(-q, min(q, exact))
        assert k[i] == exact, (w[i], s, k[i], exact)
    # ties actually occur in these sweeps and go to even
    quot = w.astype(np.float64) / float(s)
    ties = np.flatnonzero(quot - np.floor(quot) == 0.5)
    if len(ties):
        assert np.all(k[ties] % 2 == 0)


@pytest.mark.parametrize("b", [3, 4, 8])
def test_invariants_random(b):
    rng = np.random.default_rng(b)
    w = (rng.standard_normal(20000) * 0.02).astype(np.float16)
    w[123] = np.float16(-0.2)  # an outlier that becomes the absmax
    m, s, k = Qz.quantize_expert(w, b)
    q = q_levels(b)
    assert m == 0.2 or m == float(np.float16(0.2))
    assert np.all(np.abs(k) <= q)
    assert k[123] == -q
    Qw = Qz.dequantize(k, s)
    S = Fraction(float(s))
    for i in range(0, len(w), 13):
        assert abs(Fraction(float(Qw[i])) - Fraction(float(w[i]))) <= S / 2
    # Q(Q(w)) = Q(w): requantising the dequantized values (same absmax q*s,
    # same scale) returns the same codes
    m2 = float(np.max(np.abs(Qw)))
    assert m2 == q * float(s)
    s2 = np.float32(np.float64(m2) / q)
    assert s2 == s
    k2 = np.clip(np.rint(Qw / np.float64(s2)), -q, q)
    assert np.array_equal(k2, k)


def test_zero_master_gives_zero_codes():
    w = np.zeros(256, dtype=np.float16)
    m, s, k = Qz.quantize_expert(w, 4)
    assert m == 0.0 and s == 0.0 and np.all(k == 0)
    assert np.all(Qz.offset_codes(k, 4) == 8)


def test_nonfinite_master_rejected():
    w = np.zeros(8, dtype=np.float16)
    w[3] = np.float16(np.inf)
    with pytest.raises(Qz.NonFiniteMaster):
        Qz.absmax(w)
    w[3] = np.float16(np.nan)
    with pytest.raises(Qz.NonFiniteMaster):
        Qz.absmax(w)


def test_offset_codes_range():
    for b in (3, 4, 8):
        q = q_levels(b)
        u = Qz.offset_codes(np.arange(-q, q + 1), b)
        assert u.min() == 1 and u.max() == (1 << b) - 1
