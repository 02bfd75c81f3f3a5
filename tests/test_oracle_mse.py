"""Pins for the measured per-expert loss and the loss-table allocator.

PagedWeight, "Quality-Aware Quantization": L(b) is a loss such as the mean
squared error, and experts differ in sensitivity. quantization_mse measures the
mean squared error of an expert's own quantization; allocate_bits_table solves
the page's allocation problem with a loss per expert and width.

The MSE is pinned by the quantizer's hand-worked examples (errors worked out
by hand from Q(w) = round(w / s) s), by exact rational arithmetic on random
experts (fractions.Fraction, a different route to the same sum), by bounds
(|w - Q(w)| <= s / 2) and by the uniform-error closed form s^2 / 12. The
table allocator is pinned by exhaustive search over 3^E assignments.
"""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest

from oracle import allocate as A
from oracle import quantize as Q


# Hand-worked errors for the quantizer's worked examples (k from the same
# examples; error = w - k s, squared and averaged by hand):
#  b=3: s = 1/2, errors 0, 1/4, 1/4, 0, 0, 1/8       -> (9/64) / 6
#  b=4: s = 1/8, errors 0, -1/16, 1/16, 1/16, 0, 1/16 -> (1/64) / 6
#  b=8: s = 2^-7, errors 0, -2^-8, -2^-8, 0, 13/4096   -> (681/2^24) / 5
HAND = [
    (3, [1.5, -0.75, 0.25, 0.5, -1.0, 0.125], Fraction(9, 64) / 6),
    (4, [0.875, -0.3125, 0.0625, -0.1875, 0.5, -0.4375], Fraction(1, 64) / 6),
    (8, [0.9921875, -0.00390625, 0.01171875, -0.5, 0.300048828125], Fraction(681, 2 ** 24) / 5),
]


@pytest.mark.parametrize("b,w,mse", HAND)
def test_hand_worked_mse(b, w, mse):
    assert Q.quantization_mse(np.array(w, dtype=np.float16), b) == float(mse)


def exact_mse(w16, b):
    """The same quantity through Fractions: the exact quotient's rounding,
    the exact errors and their exact sum, then the two roundings."""
    w = [Fraction(float(x)) for x in w16.astype(np.float64)]
    m = max(abs(x) for x in w)
    q = (1 << (b - 1)) - 1
    s = Fraction(float(np.float32(float(m) / q))) if m != 0 else Fraction(0)
    total = Fraction(0)
    for x in w:
        if s == 0:
            k = 0
        else:
            r = x / s
            k = math.floor(r)
            frac = r - k
            if frac > Fraction(1, 2) or (frac == Fraction(1, 2) and k % 2 == 1):
                k += 1
            k = max(-q, min(q, k))
        total += (x - k * s) ** 2
    return float(np.float64(float(total)) / np.float64(len(w)))


@pytest.mark.parametrize("seed", range(8))
@pytest.mark.parametrize("b", [3, 4, 8])
def test_mse_matches_exact_rationals(seed, b):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 400))
    scale = [0.02, 3.0, 1e-5, 700.0][seed % 4]  # small, large (s >= 1), subnormal-heavy, huge
    w = (rng.standard_normal(n) * scale).astype(np.float16)
    if seed % 2 == 0:
        # half-integer quotients: weights on the half-grid of the scale
        m = float(np.max(np.abs(w.astype(np.float64))))
        if m > 0:
            s = float(np.float32(m / ((1 << (b - 1)) - 1)))
            j = rng.integers(-2 * ((1 << (b - 1)) - 1), 2 * ((1 << (b - 1)) - 1) + 1, size=n // 3)
            w[: n // 3] = (j * (s / 2)).astype(np.float16)
    assert Q.quantization_mse(w, b) == exact_mse(w, b)


@pytest.mark.parametrize("b", [3, 4, 8])
def test_mse_bounds_and_special_cases(b):
    rng = np.random.default_rng(7)
    w = (rng.standard_normal(5000) * 0.02).astype(np.float16)
    m, s, k = Q.quantize_expert(w, b)
    mse = Q.quantization_mse(w, b)
    assert 0.0 < mse <= float(s) ** 2 / 4
    assert Q.quantization_mse(np.zeros(64, np.float16), b) == 0.0
    # weights that are exact multiples of s (b = 8: k s is fp16-exact here)
    grid = (np.arange(-127, 128) * 2.0 ** -7).astype(np.float16)
    assert Q.quantization_mse(grid, 8) == 0.0


@pytest.mark.parametrize("b", [3, 4])
def test_mse_uniform_error_closed_form(b):
    # weights spread evenly over [-m, m] on a grid much finer than s: the error
    # is uniform on [-s/2, s/2], so the MSE is s^2 / 12 up to the grid
    m = 1.0
    w = np.linspace(-m, m, 20001).astype(np.float16)
    s = float(np.float32(m / ((1 << (b - 1)) - 1)))
    assert Q.quantization_mse(w, b) == pytest.approx(s * s / 12, rel=0.02)


def brute_force_table(p, L, W, B):
    best, arg = math.inf, []
    for bits in itertools.product((3, 4, 8), repeat=len(W)):
        if sum(b * w for b, w in zip(bits, W)) > B:
            continue
        v = 0.0
        for e, b in enumerate(bits):
            v = v + p[e] * L[e][(3, 4, 8).index(b)]
        if v < best:
            best, arg = v, [bits]
        elif v == best:
            arg.append(bits)
    return best, arg


@pytest.mark.parametrize("seed", range(16))
def test_table_dp_matches_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    E = int(rng.integers(1, 8))
    p = rng.dirichlet(np.full(E, 0.6))
    # losses per expert; some rows are not decreasing in b
    L = rng.uniform(1e-6, 1e-2, size=(E, 3))
    if seed % 3 == 0:
        L = np.sort(L, axis=1)[:, ::-1].copy()
    W = [int(x) for x in rng.choice([1024, 2048, 3072], size=E)] if seed % 2 else [4096] * E
    sw = sum(W)
    B = int(rng.integers(3 * sw, 9 * sw + 1))
    bits = A.allocate_bits_table(p, L, W, B)
    best, args = brute_force_table(p, L, W, B)
    assert A.objective_table(p, L, bits) == best
    assert tuple(int(b) for b in bits) in args
    assert A.budget_used(W, bits) <= B


def test_table_with_constant_rows_is_the_fixed_loss_program():
    rng = np.random.default_rng(5)
    E = 12
    p = rng.dirichlet(np.ones(E))
    W = [2048] * E
    rows = np.tile([A.loss(3), A.loss(4), A.loss(8)], (E, 1))
    for avg in (3.0, 3.4, 4.5, 6.0, 7.9):
        B = int(avg * sum(W))
        assert (A.allocate_bits_table(p, rows, W, B) == A.allocate_bits(p, W, B)).all()


def test_table_errors_and_unlimited_budget():
    p = np.array([0.5, 0.5, 0.0])
    L = np.array([[3e-3, 1e-3, 1e-5], [3e-3, 4e-3, 1e-5], [1.0, 0.5, 0.1]])
    W = [256, 256, 256]
    with pytest.raises(A.Infeasible):
        A.allocate_bits_table(p, L, W, 3 * 768 - 1)
    with pytest.raises(ValueError):
        A.allocate_bits_table(p, L[:2], W, 8 * 768)
    # unlimited budget: each expert takes its least cost, ties (p = 0) the lowest width
    assert list(A.allocate_bits_table(p, L, W, 8 * 768)) == [8, 8, 3]
