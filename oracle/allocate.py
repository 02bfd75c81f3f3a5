"""Budgeted per-expert precision: the exact solution of PagedWeight's allocation problem.

PagedWeight, "Quality-Aware Quantization": choose b_e to minimise
sum_e p_e * L(b_e) subject to sum_e b_e * W_e <= B, where p_e is the expert's
average routing probability and W_e its number of weight elements. The bit
widths available are {3, 4, 8} (PagedWeight, "Code Illustration", bit_options).

Readings taken where the page is open:
* L(b) is the mean squared error of a uniform symmetric quantizer whose step
  is proportional to 1/q_b, q_b = 2^(b-1) - 1, so L(b) = 1 / q_b^2 (the page
  says "e.g., mean squared error"; the allocator receives no weights, so the
  loss is expert-independent up to p_e).
* B counts bits of codes only (scales and page slack are not counted), as in
  the page's constraint.
* The problem is solved exactly (dynamic program), not by the page's
  simplified proportional illustration.

Dynamic program (units of g = gcd(W_e)): R = floor((B - 3*sum W) / g) budget
units may be spent on upgrades; upgrading expert e from 3 to 4 bits costs
W_e/g units, from 3 to 8 bits 5*W_e/g. D_e[r] is the least objective over the
first e experts that spend exactly r units. Options are tried in the order
3, 4, 8 and replace the incumbent only when strictly smaller (ties keep the
lower width). The answer is argmin_r D_E[r] (ties: smallest r), then a
backtrack. Costs are p_e * L(b) (one float64 multiply) added to D_{e-1}
(one float64 add), with no fused multiply-add.
"""
from __future__ import annotations

import math

import numpy as np

BIT_OPTIONS = (3, 4, 8)


class Infeasible(ValueError):
    """B < 3 * sum_e W_e: even all-3-bit experts exceed the budget."""


class StateCapExceeded(ValueError):
    """The budget, in units of gcd(W_e), needs more DP states than the cap allows."""


def q_levels(b: int) -> int:
    """q_b = 2^(b-1) - 1, the largest code magnitude at b bits."""
    return (1 << (b - 1)) - 1


def loss(b: int) -> float:
    """L(b) = 1 / q_b^2 in float64."""
    q = q_levels(b)
    return 1.0 / float(q * q)


def allocate_bits(p, W, B: int, state_cap: int = 1 << 22) -> np.ndarray:
    """b_e in {3,4,8} minimising sum p_e L(b_e) under sum b_e W_e <= B.

    p: float64[E] importances; W: int[E] weight elements (> 0); B: budget in bits.
    Returns uint8[E]. Raises Infeasible or StateCapExceeded.
    """
    E = len(W)
    if E > 0 and len(p) == E and all(int(w) > 0 for w in W) and int(B) >= 8 * sum(int(w) for w in W):
        return np.full(E, 8, dtype=np.uint8)
    table = np.tile(np.array([loss(b) for b in BIT_OPTIONS], dtype=np.float64), (E, 1))
    return allocate_bits_table(p, table, W, B, state_cap)


def allocate_bits_table(p, L, W, B: int, state_cap: int = 1 << 22) -> np.ndarray:
    """The same program with a loss per expert and width: minimise
    sum_e p_e L[e, b_e] under sum b_e W_e <= B, L float64[E, 3] with columns
    for 3, 4 and 8 bits. With every row (1/9, 1/49, 1/16129) this is
    allocate_bits; with L[e] the measured quantization error of expert e
    (quantize.quantization_mse) it is the page's "sensitivity" reading of
    L_e(b). Each cost p_e * L[e, b] is one float64 multiply.
    """
    p = np.asarray(p, dtype=np.float64)
    L = np.asarray(L, dtype=np.float64)
    W = [int(w) for w in W]
    E = len(W)
    if E == 0 or len(p) != E or any(w <= 0 for w in W):
        raise ValueError("need E > 0 experts with W_e > 0 and one p_e each")
    if L.shape != (E, len(BIT_OPTIONS)):
        raise ValueError("need one loss row (3, 4, 8 bits) per expert")
    B = int(B)
    sum_w = sum(W)
    if B < 3 * sum_w:
        raise Infeasible(f"B={B} < 3*sum(W)={3 * sum_w}")
    # a budget of 8 sum W or more caps R at every expert's 3 -> 8 upgrade; the
    # program then picks each expert's least p_e L[e, b] (all 8 for allocate_bits,
    # which returns that case before coming here)
    g = 0
    for w in W:
        g = math.gcd(g, w)
    up = [{3: 0, 4: w // g, 8: 5 * w // g} for w in W]
    R = (B - 3 * sum_w) // g
    R = min(R, sum(u[8] for u in up))
    if R + 1 > state_cap:
        raise StateCapExceeded(f"{R + 1} states > cap {state_cap}")

    inf = math.inf
    D = [0.0] + [inf] * R
    choice = np.zeros((E, R + 1), dtype=np.uint8)
    for e in range(E):
        Dn = [inf] * (R + 1)
        for r in range(R + 1):
            best = inf
            best_b = 0
            for i, b in enumerate(BIT_OPTIONS):
                rp = r - up[e][b]
                if rp < 0:
                    continue
                prev = D[rp]
                if prev == inf:
                    continue
                cost = p[e] * L[e, i]       # float64 multiply
                cand = prev + cost          # float64 add
                if cand < best:
                    best = cand
                    best_b = b
            Dn[r] = best
            choice[e, r] = best_b
        D = Dn

    r_best = 0
    for r in range(1, R + 1):
        if D[r] < D[r_best]:
            r_best = r
    bits = np.zeros(E, dtype=np.uint8)
    r = r_best
    for e in range(E - 1, -1, -1):
        b = int(choice[e, r])
        assert b in BIT_OPTIONS
        bits[e] = b
        r -= up[e][b]
    assert r == 0
    return bits


def objective(p, bits) -> float:
    """sum_e p_e L(b_e), accumulated in ascending e with float64 multiply then add."""
    total = 0.0
    for pe, b in zip(np.asarray(p, dtype=np.float64), bits):
        total = total + pe * loss(int(b))
    return total


def objective_table(p, L, bits) -> float:
    """sum_e p_e L[e, b_e], ascending e, float64 multiply then add."""
    L = np.asarray(L, dtype=np.float64)
    total = 0.0
    for e, (pe, b) in enumerate(zip(np.asarray(p, dtype=np.float64), bits)):
        total = total + pe * L[e, BIT_OPTIONS.index(int(b))]
    return total


def budget_used(W, bits) -> int:
    return sum(int(w) * int(b) for w, b in zip(W, bits))


def proportional_widths(p, W, B: int) -> np.ndarray:
    """The page's simplified allocator ("Code Illustration",
    compute_budgeted_precision), read for what it computes: expert e gets the
    budget share B p_e / sum p, i.e. share / W_e bits per weight, rounded UP to
    the next available width (3 if at most 3, 4 if in (3, 4], 8 above 4 -- the
    illustration's bucketize over (3, 4, 8) with the index clamped to the last
    width). The result can exceed the budget.

    Float64, in this order: total = p_0 + p_1 + ... (ascending e); share =
    (B * p_e) / total; bits = share / W_e. B counts bits (the illustration's
    "budget_bytes" divided by element counts is read as bits per element, as in
    the exact allocator); all-zero importances give every expert 3 bits.
    """
    p = np.asarray(p, dtype=np.float64)
    W = [int(w) for w in W]
    E = len(W)
    if E == 0 or len(p) != E or any(w <= 0 for w in W):
        raise ValueError("need E > 0 experts with W_e > 0 and one p_e each")
    total = 0.0
    for pe in p:
        total = total + float(pe)
    bits = np.empty(E, dtype=np.uint8)
    for e in range(E):
        share = (float(int(B)) * float(p[e])) / total if total > 0.0 else 0.0
        per_weight = share / float(W[e])
        bits[e] = 3 if per_weight <= 3.0 else (4 if per_weight <= 4.0 else 8)
    return bits


def allocate_bits_proportional(p, W, B: int) -> np.ndarray:
    """proportional_widths followed by a budget repair -- a reading of this
    build (the illustration has no such step): experts are walked in ascending
    (p_e, e) and each is downgraded one width at a time (8 -> 4 -> 3) until
    sum b_e W_e <= B. Raises Infeasible if B < 3 sum W."""
    W = [int(w) for w in W]
    B = int(B)
    if B < 3 * sum(W):
        raise Infeasible(f"B={B} < 3*sum(W)={3 * sum(W)}")
    p = np.asarray(p, dtype=np.float64)
    bits = proportional_widths(p, W, B)
    used = budget_used(W, bits)
    for e in sorted(range(len(W)), key=lambda i: (float(p[i]), i)):
        if used <= B:
            break
        if bits[e] == 8:
            bits[e] = 4
            used -= 4 * W[e]
        if used <= B:
            break
        if bits[e] == 4:
            bits[e] = 3
            used -= W[e]
    assert used <= B
    return bits
