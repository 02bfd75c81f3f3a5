"""Pins for oracle.allocate (PagedWeight, "Quality-Aware Quantization").

The dynamic program is checked against exhaustive search over all 3^E width
assignments (a different algorithm that evaluates the page's objective and
constraint directly), against the special cases the constraint fixes, and
against the exchange property of the optimum for equal-size experts.
"""
import itertools
import math

import numpy as np
import pytest

from oracle import allocate as A


def brute_force(p, W, B):
    """Exhaustive min of sum p_e L(b_e) over {3,4,8}^E with sum b_e W_e <= B.

    The objective is accumulated in ascending e (same float64 order as the DP),
    so the optimal value compares exactly. Returns (best value, all optimal
    assignments)."""
    Ls = {b: 1.0 / float(((1 << (b - 1)) - 1) ** 2) for b in (3, 4, 8)}
    best, arg = math.inf, []
    for bits in itertools.product((3, 4, 8), repeat=len(W)):
        if sum(b * w for b, w in zip(bits, W)) > B:
            continue
        v = 0.0
        for pe, b in zip(p, bits):
            v = v + pe * Ls[b]
        if v < best:
            best, arg = v, [bits]
        elif v == best:
            arg.append(bits)
    return best, arg


def test_loss_values():
    # L(b) = 1/q_b^2, q_b = 2^(b-1)-1: q = 3, 7, 127
    assert A.q_levels(3) == 3 and A.q_levels(4) == 7 and A.q_levels(8) == 127
    assert A.loss(3) == 1.0 / 9.0
    assert A.loss(4) == 1.0 / 49.0
    assert A.loss(8) == 1.0 / 16129.0


@pytest.mark.parametrize("seed", range(12))
def test_dp_matches_brute_force_equal_W(seed):
    rng = np.random.default_rng(seed)
    E = int(rng.integers(1, 9))
    p = rng.dirichlet(np.full(E, 0.7))
    W = [393216] * E
    sw = sum(W)
    B = int(rng.integers(3 * sw, 8 * sw + 1))
    bits = A.allocate_bits(p, W, B)
    best, args = brute_force(p, W, B)
    assert A.objective(p, bits) == best
    assert tuple(int(b) for b in bits) in args
    assert A.budget_used(W, bits) <= B


@pytest.mark.parametrize("seed", range(12))
def test_dp_matches_brute_force_unequal_W(seed):
    rng = np.random.default_rng(100 + seed)
    E = int(rng.integers(1, 8))
    p = rng.dirichlet(np.full(E, 1.0))
    W = [int(x) * 64 for x in rng.integers(1, 40, size=E)]
    sw = sum(W)
    B = int(rng.integers(3 * sw, 8 * sw + 1))
    bits = A.allocate_bits(p, W, B)
    best, args = brute_force(p, W, B)
    assert A.objective(p, bits) == best
    assert tuple(int(b) for b in bits) in args


def test_tiny_layer_budget_brute_force():
    # 8 experts of 3*256*512 weights at 4.5 bits average: 3^8 = 6561 assignments
    rng = np.random.default_rng(7)
    p = rng.dirichlet(np.ones(8))
    W = [3 * 256 * 512] * 8
    B = int(math.floor(4.5 * sum(W)))
    bits = A.allocate_bits(p, W, B)
    best, args = brute_force(p, W, B)
    assert A.objective(p, bits) == best and tuple(int(b) for b in bits) in args
    assert len(set(int(b) for b in bits)) >= 2  # a mixed allocation


def test_special_cases():
    p = np.array([0.5, 0.3, 0.2])
    W = [100, 200, 300]
    sw = sum(W)
    assert list(A.allocate_bits(p, W, 3 * sw)) == [3, 3, 3]
    assert list(A.allocate_bits(p, W, 8 * sw)) == [8, 8, 8]
    assert list(A.allocate_bits(p, W, 10 * sw)) == [8, 8, 8]
    with pytest.raises(A.Infeasible):
        A.allocate_bits(p, W, 3 * sw - 1)


def test_single_expert_takes_widest_that_fits():
    W = [1000]
    assert list(A.allocate_bits([1.0], W, 3999)) == [3]
    assert list(A.allocate_bits([1.0], W, 4000)) == [4]
    assert list(A.allocate_bits([1.0], W, 7999)) == [4]
    assert list(A.allocate_bits([1.0], W, 8000)) == [8]


def test_zero_importance_gets_lowest_width():
    # an expert with p_e = 0 gains nothing from bits: ties keep 3 bits
    bits = A.allocate_bits([0.0, 1.0], [10, 10], 8 * 20 - 1)
    assert list(bits) == [3, 8]


def test_equal_experts_tie_in_expert_order():
    # Two experts with equal p and W: giving the upgrade to either costs the
    # same (p L(4) + p L(3) = p L(3) + p L(4) exactly, the sum commutes). The
    # program tries 3, 4, 8 in that order and replaces its best only on a
    # strictly smaller cost, so the later expert keeps the lower width and the
    # earlier one takes the upgrade. Budget units of W = 10 bits: one unit
    # buys 3 -> 4, five buy 3 -> 8.
    W = [10, 10]
    assert list(A.allocate_bits([0.5, 0.5], W, 3 * 20 + 10)) == [4, 3]
    # six units: 8 + 4 either way (L(8) + L(4) beats 4 + 4 and 8 + 3)
    assert list(A.allocate_bits([0.5, 0.5], W, 3 * 20 + 60)) == [8, 4]


@pytest.mark.parametrize("seed", range(6))
def test_exchange_property_equal_W(seed):
    # for equal W_e, swapping widths between i and j keeps the budget; an optimum
    # therefore never gives the more important expert fewer bits
    rng = np.random.default_rng(200 + seed)
    E = 64
    p = rng.dirichlet(np.full(E, 0.5))
    W = [4718592] * E
    B = int(math.floor(3.5 * sum(W)))
    bits = A.allocate_bits(p, W, B)
    assert A.budget_used(W, bits) <= B
    for i in range(E):
        for j in range(E):
            if p[i] > p[j]:
                assert bits[i] >= bits[j]


def test_state_cap():
    with pytest.raises(A.StateCapExceeded):
        A.allocate_bits([0.5, 0.5], [1, 2], 3 * 3 + 10, state_cap=4)


# ----------------------------------------------------------------------------
# the page's proportional illustration (+ budget repair), a selectable variant
# ----------------------------------------------------------------------------
def test_proportional_rounds_up_like_the_illustration():
    # one expert, so its share is the whole budget: B / W bits a weight, rounded
    # up to the next width (3.0 -> 3, 3.001 -> 4, 4.0 -> 4, 4.001 -> 8, > 8 -> 8)
    # (p = 0.5 keeps B p / p exact in float64; p = 0.7 would give 4000.0000000000005)
    W = [1000]
    cases = {1000: 3, 3000: 3, 3001: 4, 3010: 4, 4000: 4, 4001: 8, 4500: 8, 8000: 8, 9000: 8}
    for B, want in cases.items():
        assert list(A.proportional_widths([0.5], W, B)) == [want], B
    # the repair then brings a width that exceeds the budget down
    assert list(A.allocate_bits_proportional([0.5], W, 3001)) == [3]
    assert list(A.allocate_bits_proportional([0.5], W, 4500)) == [4]
    assert list(A.allocate_bits_proportional([0.5], W, 9000)) == [8]
    # all-zero importances: no share, 3 bits
    assert list(A.proportional_widths([0.0, 0.0], [10, 10], 100)) == [3, 3]


def test_proportional_hand_example():
    # shares 160/320/480/640 bits for W = 100: 1.6, 3.2, 4.8, 6.4 bits a weight
    # -> (3, 4, 8, 8) using 2300 > 1600; repair in ascending p: expert 1 4->3
    # (2200), expert 2 8->4 (1800) and 4->3 (1700), expert 3 8->4 (1300)
    p = [0.1, 0.2, 0.3, 0.4]
    bits = A.allocate_bits_proportional(p, [100] * 4, 1600)
    assert list(bits) == [3, 3, 3, 4]
    # a budget that fits the rounded-up widths is left alone
    assert list(A.allocate_bits_proportional(p, [100] * 4, 2300)) == [3, 4, 8, 8]


def test_proportional_budget_and_errors():
    rng = np.random.default_rng(5)
    for _ in range(200):
        E = int(rng.integers(1, 12))
        p = rng.dirichlet(np.full(E, 0.5))
        W = [int(x) for x in rng.integers(1, 60, size=E)]
        B = int(rng.integers(3 * sum(W), 9 * sum(W)))
        bits = A.allocate_bits_proportional(p, W, B)
        assert set(bits.tolist()) <= {3, 4, 8}
        assert A.budget_used(W, bits) <= B
        # the exact allocator is never worse on the page's objective
        exact = A.allocate_bits(p, W, B)
        assert A.objective(p, exact) <= A.objective(p, bits) * (1 + 1e-12)
    with pytest.raises(A.Infeasible):
        A.allocate_bits_proportional([1.0, 1.0], [5, 5], 29)
