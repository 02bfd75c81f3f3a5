"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of an oracle function -- a dropped or
altered term, a wrong rounding, sign, index, order or tie rule -- by editing
one snippet of the function's own source, swaps it into the oracle module
(on the CPU, for this test only) and runs the pins that guard that function:
at least one of them must fail. A mistake no pin catches would let the
oracle drift from the pages unnoticed.
"""
import inspect
import textwrap

import numpy as np
import pytest

from oracle import allocate as A
from oracle import compensate as C
from oracle import ffn as Fn
from oracle import layout as L
from oracle import pages as P
from oracle import prefix as X
from oracle import quantize as Qz
from oracle import route as Rt

import test_oracle_allocate as TA
import test_oracle_compensate as TC
import test_oracle_layout_pages as TL
import test_oracle_mse as TM
import test_oracle_prefix as TX
import test_oracle_quantize as TQ
import test_oracle_route_ffn as TR


def _mutant(owner, name, old, new):
    """owner.name recompiled from its source with `old` replaced by `new`
    (exactly one occurrence), in the namespace of the oracle module that
    defines it."""
    fn = getattr(owner, name)
    src = textwrap.dedent(inspect.getsource(fn))
    assert src.count(old) == 1, (name, old)
    mod = inspect.getmodule(fn)
    ns = dict(vars(mod))
    exec(compile(src.replace(old, new), f"<mutant of {mod.__name__}.{name}>", "exec"), ns)
    return ns[name]


def _hand_quantize():
    for case in TQ.HAND:
        TQ.test_hand_worked_example(*case)


def _hand_mse():
    for case in TM.HAND:
        TM.test_hand_worked_mse(*case)


def _route_pins():
    for seed in range(8):
        TR.test_route_brute_force(seed)
    TR.test_route_properties_all_one_expert()
    TR.test_invalid_ids_contribute_nothing()


def _ffn_pins():
    TR.test_expert_ffn_triple_loop()
    TR.test_moe_ffn_loop_combine()
    TR.test_one_hot_token_reads_gate_column()
    TR.test_combine_is_linear_in_topk_weights()


def _allocate_pins():
    TA.test_loss_values()
    for seed in range(12):
        TA.test_dp_matches_brute_force_equal_W(seed)
        TA.test_dp_matches_brute_force_unequal_W(seed)
    TA.test_tiny_layer_budget_brute_force()
    TA.test_special_cases()
    TA.test_single_expert_takes_widest_that_fits()
    TA.test_zero_importance_gets_lowest_width()
    TA.test_equal_experts_tie_in_expert_order()


def _proportional_pins():
    TA.test_proportional_rounds_up_like_the_illustration()
    TA.test_proportional_hand_example()
    TA.test_proportional_budget_and_errors()


def _layout_pins():
    TL.test_hand_words_b4()
    TL.test_hand_words_b8()
    TL.test_hand_words_b3()
    for b in (3, 4, 8):
        TL.test_matrix_element_locations(b)
    TL.test_expert_stream_order()


def _page_pins():
    TL.test_allocator_hand_example()
    for seed in range(4):
        TL.test_allocator_invariants_random(seed)
    TL.test_overlapped_repage_keeps_old_pages_until_commit()


def _prefix_pins():
    TX.test_hand_worked_codes()
    TX.test_every_fp16_weight_lies_in_its_bins(1.0)
    TX.test_layers_compose_the_codes()
    TX.test_layer_b_hand_word()


def _compensate_pins():
    TC.test_salient_channels_brute_force()
    TC.test_hand_worked_linear()
    TC.test_linear_equals_mask_matrix()


def _compensate_layer_pins():
    _compensate_pins()
    TC.test_layer_ends()


MUTANTS = [
    # quantizer: PagedWeight, "Implementation Details" (s = max|w| / (2^(b-1) - 1), round)
    ("scale: q_b off by one", Qz, "scale", "np.float64(q_levels(b))",
     "np.float64(q_levels(b) + 1)", _hand_quantize),
    ("encode: ties away from zero", Qz, "encode", "np.rint(w / s64)",
     "np.sign(w) * np.floor(np.abs(w / s64) + 0.5)", _hand_quantize),
    ("encode: truncation", Qz, "encode", "np.rint(w / s64)", "np.trunc(w / s64)",
     _hand_quantize),
    ("absmax: signed max", Qz, "absmax", "np.max(np.abs(w.astype(np.float64)))",
     "np.max(w.astype(np.float64))", lambda: [TQ.test_invariants_random(b) for b in (3, 4, 8)]),
    ("offset codes: wrong offset", Qz, "offset_codes", "(1 << (b - 1))", "(1 << b)",
     TQ.test_offset_codes_range),
    ("mse: n - 1", Qz, "quantization_mse", "np.float64(sum_sq) / np.float64(n)",
     "np.float64(sum_sq) / np.float64(n - 1)", _hand_mse),
    # allocator: PagedWeight, "Quality-Aware Quantization"
    ("loss: 1/q instead of 1/q^2", A, "loss", "1.0 / float(q * q)", "1.0 / float(q)",
     _allocate_pins),
    ("DP: 8-bit upgrade costs 4 W", A, "allocate_bits_table", "8: 5 * w // g",
     "8: 4 * w // g", _allocate_pins),
    ("DP: ties take the wider width", A, "allocate_bits_table", "if cand < best:",
     "if cand <= best:", _allocate_pins),
    ("DP: budget tie to the largest", A, "allocate_bits_table", "if D[r] < D[r_best]:",
     "if D[r] <= D[r_best]:", _allocate_pins),
    ("DP: cost without the importance", A, "allocate_bits_table", "cost = p[e] * L[e, i]",
     "cost = L[e, i]", _allocate_pins),
    ("proportional: 3-bit edge open", A, "proportional_widths", "per_weight <= 3.0",
     "per_weight < 3.0", _proportional_pins),
    ("proportional: share not normalised", A, "proportional_widths",
     "(float(int(B)) * float(p[e])) / total", "float(int(B)) * float(p[e])",
     _proportional_pins),
    # routing: PagedWeight, "Dynamic Paging" (tokens bucketed by expert)
    ("route: unstable order", Rt, "route", 'kind="stable"', 'kind="quicksort"', _route_pins),
    ("route: inclusive offsets", Rt, "route", "offsets[1:] = np.cumsum(counts)",
     "offsets[:-1] = np.cumsum(counts)", _route_pins),
    ("route: dropped ids map to 0", Rt, "route", "inv = np.full(ids.size, -1",
     "inv = np.full(ids.size, 0", _route_pins),
    ("route: id E accepted", Rt, "route", "valid = (ids >= 0) & (ids < E)",
     "valid = (ids >= 0) & (ids <= E)", _route_pins),
    # FFN: SwiGLU from the dequantized weights
    ("ffn: gate and up swapped", Fn, "expert_ffn", "h = silu(g) * v", "h = silu(v) * g",
     _ffn_pins),
    ("ffn: no activation", Fn, "expert_ffn", "h = silu(g) * v", "h = g * v", _ffn_pins),
    ("ffn: sigmoid sign", Fn, "silu", "np.exp(-g)", "np.exp(g)", _ffn_pins),
    ("ffn: down transposed", Fn, "expert_ffn", "return h @ w2.T", "return h @ w2",
     _ffn_pins),
    ("combine: first slot's weight", Fn, "moe_ffn", "out[oi] += w[t, j] * y[r]",
     "out[oi] += w[t, 0] * y[r]", _ffn_pins),
    # packed format and pages: PagedWeight, "Dynamic Paging"
    ("layout: 4-bit fields not interleaved", L, "_shifts",
     "np.array([16 * (i & 1) + 4 * (i >> 1) for i in range(8)]", "np.array([4 * i for i in range(8)]",
     _layout_pins),
    ("layout: gate/up chunks not interleaved", L, "expert_stream",
     "gu = np.stack([g1, g3], axis=1)", "gu = np.stack([g1, g3], axis=0)", _layout_pins),
    ("layout: 3-bit code 31 in bit 30", L, "pack_quarters",
     "& np.uint32(1)) << np.uint32(31)", "& np.uint32(1)) << np.uint32(30)", _layout_pins),
    ("layout: 3-bit fields not interleaved", L, "_shifts",
     "np.array([16 * (i & 1) + 3 * (i >> 1) for i in range(10)]",
     "np.array([3 * i for i in range(10)]", _layout_pins),
    ("layout: down tiles not paired", L, "expert_stream", "g2.transpose(0, 2, 1, 3)",
     "g2.transpose(0, 1, 2, 3)", _layout_pins),
    ("pages: highest free page first", P.PageAllocator, "_take",
     "idx = np.flatnonzero(free)[:n]", "idx = np.flatnonzero(free)[::-1][:n]", _page_pins),
    ("pages: table offsets past the expert", P.PageAllocator, "table",
     "first[e] = len(idx)", "first[e] = len(idx) + len(self.pages[e])", _page_pins),
    ("pages: repage keeps the old pages", P.PageAllocator, "repage",
     "free[pages[e]] = True", "pass", _page_pins),
    ("pages: overlapped repage frees at once", P.PageAllocator, "repage_overlapped",
     "released.extend(pages[e])", "free[pages[e]] = True", _page_pins),
    ("proportional: repair from the most important", A, "allocate_bits_proportional",
     "key=lambda i: (float(p[i]), i)", "key=lambda i: (-float(p[i]), i)", _proportional_pins),
    # prefix-compatible grid
    ("prefix: rounding instead of floor", X, "prefix_codes", "u8 = (128 * wi) // mi + 128",
     "u8 = np.rint(128 * wi / mi).astype(np.int64) + 128", _prefix_pins),
    ("prefix: layer B from the wrong bit", X, "layer_values", '"B": (u8 >> 4) & 1',
     '"B": (u8 >> 3) & 1', _prefix_pins),
    ("prefix: bin edge instead of centre", X, "dequantize",
     "(2.0 * np.asarray(u_b, dtype=np.float64) + 1.0 - float(1 << b))",
     "(2.0 * np.asarray(u_b, dtype=np.float64) - float(1 << b))", _prefix_pins),
    # compensation: DecDEC summary, 3.1-3.2 (channels by activation magnitude)
    ("compensation: smallest channels", C, "salient_channels", "-np.abs(row)", "np.abs(row)",
     _compensate_pins),
    ("compensation: down from the plain gate", C, "expert_ffn_compensated",
     "g = compensated_linear(w1h, w1, x, n)", "g = w1h @ x", _compensate_layer_pins),
    ("compensation: residual sign", C, "compensated_linear",
     "(w[:, sel] - w_hat[:, sel]) @ x[sel]", "(w_hat[:, sel] - w[:, sel]) @ x[sel]",
     _compensate_pins),
    ("compensation: ties to the higher index", C, "salient_channels",
     "np.lexsort((np.arange(L), -np.abs(row)))", "np.lexsort((-np.arange(L), -np.abs(row)))",
     _compensate_pins),
]


@pytest.mark.parametrize("label,owner,name,old,new,pins", MUTANTS,
                         ids=[m[0] for m in MUTANTS])
def test_pins_catch_the_planted_mistake(monkeypatch, label, owner, name, old, new, pins):
    pins()  # the pins pass on the oracle as it is
    monkeypatch.setattr(owner, name, _mutant(owner, name, old, new))
    with pytest.raises(Exception):
        pins()
