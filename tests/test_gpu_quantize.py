"""GPU parity for the allocator, the absmax quantizer, the packer and the page
table: bit-exact against the float64 oracle (PagedWeight, "Quality-Aware
Quantization" and "Implementation Details")."""
import numpy as np
import pytest
import torch

import synth
from oracle import allocate as oa
from oracle import pages as op

from _helpers import OracleExpert

pytestmark = pytest.mark.gpu

mpe = pytest.importorskip("mixed_precision_expert_b200")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixed_precision_expert_b200.build import build
    build()
    assert torch.cuda.is_available()


@pytest.mark.parametrize("seed", range(10))
def test_allocate_bits_small(seed):
    rng = np.random.default_rng(seed)
    E = int(rng.integers(1, 9))
    p = rng.dirichlet(np.full(E, 0.6))
    W = [int(x) * 128 for x in rng.integers(1, 50, size=E)]
    B = int(rng.integers(3 * sum(W), 8 * sum(W) + 10))
    got = mpe.allocate_bits(p, W, B)
    ref = oa.allocate_bits(p, W, B, state_cap=mpe.ALLOC_STATE_CAP)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("E,units", [(2, 1), (2, 6), (5, 3), (8, 13)])
def test_allocate_bits_ties_follow_expert_order(E, units):
    # equal importances and sizes: an upgrade costs the same whichever expert
    # takes it, up to the rounding of the running sums, so the tie rule
    # (widths tried 3, 4, 8, replaced only on a strictly smaller cost; the
    # budget argmin ties to the smallest state) and the order of the float64
    # additions decide; `units` of 128 bits buy 3 -> 4 (one) or 3 -> 8 (five)
    W = [128] * E
    p = np.full(E, 1.0 / E)
    B = 3 * sum(W) + units * 128
    got = mpe.allocate_bits(p, W, B)
    ref = oa.allocate_bits(p, W, B, state_cap=mpe.ALLOC_STATE_CAP)
    assert np.array_equal(got, ref)
    if (E, units) == (2, 1):
        assert list(got) == [4, 3]


@pytest.mark.parametrize("cfg,avg", [(1, 4.5), (2, 4.5), (3, 3.5), (5, 8.0), (5, 6.0), (5, 3.0),
                                     (5, 3.75), (5, 5.25), (3, 3.0), (3, 7.99)])
def test_allocate_bits_workloads(cfg, avg):
    wl = synth.WORKLOADS[cfg]
    p = synth.importance(wl)
    W = [wl.W_e] * wl.E
    B = synth.budget_for(wl, avg)
    got = mpe.allocate_bits(p, W, B)
    ref = oa.allocate_bits(p, W, B, state_cap=mpe.ALLOC_STATE_CAP)
    assert np.array_equal(got, ref)
    assert sum(int(b) * w for b, w in zip(got, W)) <= B


@pytest.mark.parametrize("units", [9000, 12000])
def test_allocate_bits_many_states(units):
    # sizes with gcd 1 give about `units` budget states: at 9000 the DP rows and
    # the 2-bit choice table fit in the kernel's shared memory, at 12000 they
    # live in global memory
    rng = np.random.default_rng(units)
    E = 16
    W = [int(x) for x in rng.integers(3000, 5000, size=E)]
    W[0] = 4099  # prime: gcd(W) = 1
    p = rng.dirichlet(np.full(E, 0.7))
    B = 3 * sum(W) + units
    got = mpe.allocate_bits(p, W, B)
    ref = oa.allocate_bits(p, W, B, state_cap=mpe.ALLOC_STATE_CAP)
    assert np.array_equal(got, ref)
    assert sum(int(b) * w for b, w in zip(got, W)) <= B


def test_allocate_bits_errors():
    with pytest.raises(mpe.MpeError) as ei:
        mpe.allocate_bits([1.0, 1.0], [7, 11], 3 * 18 - 1)
    assert ei.value.code == -2
    with pytest.raises(mpe.MpeError) as ei:
        mpe.allocate_bits([0.5, 0.5], [1, 100000], 3 * 100001 + 70000)
    assert ei.value.code == -3
    assert list(mpe.allocate_bits([0.2, 0.8], [5, 5], 80)) == [8, 8]


def _check_expert_state(ctx, wl, bits, masters_cpu, alloc):
    E, H, F = wl.E, wl.H, wl.F
    scales, absmax = ctx.scales()
    pte, pidx = ctx.page_table()
    table = alloc.table()
    assert np.array_equal(pte["bits"], np.asarray(bits, np.uint8))
    assert np.array_equal(pte["first"], table.first)
    assert np.array_equal(pte["n_pages"], table.n_pages)
    assert np.array_equal(pidx, table.page_idx)
    for e in range(E):
        ox = OracleExpert(masters_cpu[e], H, F, int(bits[e]))
        assert absmax[e] == np.float32(ox.m), e
        assert scales[e] == ox.s, (e, scales[e], ox.s)
        got = ctx.expert_stream(e)
        ref = ox.stream()
        assert got.size == ref.size == int(bits[e]) * wl.W_e // 8
        assert np.array_equal(got, ref), f"expert {e}: {np.flatnonzero(got != ref)[:8]}"


def test_quantize_tiny_layer():
    wl = synth.WORKLOADS[1]
    p = synth.importance(wl)
    bits = mpe.allocate_bits(p, [wl.W_e] * wl.E, wl.budget_bits)
    assert len(set(bits.tolist())) >= 2
    masters = [synth.expert_weights(wl, e, device="cuda") for e in range(wl.E)]
    cpu = [m.cpu().numpy() for m in masters]
    ctx = mpe.Context(wl.E, wl.H, wl.F)
    ctx.quantize_experts(masters, bits)
    alloc = op.PageAllocator(wl.E * op.pages_needed(8, wl.H, wl.F), wl.E, wl.H, wl.F)
    alloc.place(bits)
    _check_expert_state(ctx, wl, bits, cpu, alloc)
    assert ctx.status() == 0


@pytest.mark.parametrize("page_bytes", [4096, 12288])
def test_quantize_small_pages_every_width(page_bytes):
    # small pages: chunks of one expert spread over many pages
    wl = synth.scaled(synth.WORKLOADS[1], E=6, H=256, F=384)
    bits = np.array([3, 4, 8, 8, 3, 4], np.uint8)
    masters = [synth.expert_weights(wl, e, device="cuda") for e in range(wl.E)]
    cpu = [m.cpu().numpy() for m in masters]
    pool = 400  # 274 pages at 4 KiB: 29 + 36 + 72 + 72 + 29 + 36
    ctx = mpe.Context(wl.E, wl.H, wl.F, page_bytes=page_bytes, pool_pages=pool)
    ctx.quantize_experts(masters, bits)
    alloc = op.PageAllocator(pool, wl.E, wl.H, wl.F, page_bytes=page_bytes)
    alloc.place(bits)
    _check_expert_state(ctx, wl, bits, cpu, alloc)


def test_zero_and_nonfinite_masters():
    wl = synth.scaled(synth.WORKLOADS[1], E=3, H=128, F=128)
    masters = [synth.expert_weights(wl, e, device="cuda") for e in range(3)]
    masters[1].zero_()
    masters[2][12345] = float("nan")
    bits = np.array([4, 3, 8], np.uint8)
    ctx = mpe.Context(3, 128, 128)
    ctx.quantize_experts(masters, bits)
    st = ctx.status(clear=True)
    assert st & mpe.STATUS_NONFINITE
    s, m = ctx.scales()
    assert s[1] == 0.0 and m[1] == 0.0
    assert np.isnan(s[2])
    z = OracleExpert(masters[1].cpu().numpy(), 128, 128, 3)
    assert np.array_equal(ctx.expert_stream(1), z.stream())  # all codes = 4 (k = 0)
    o = OracleExpert(masters[0].cpu().numpy(), 128, 128, 4)
    assert np.array_equal(ctx.expert_stream(0), o.stream())


def test_repage_schedule_matches_oracle():
    wl = synth.scaled(synth.WORKLOADS[1], E=8, H=256, F=256)
    p = synth.importance(wl)
    W = [wl.W_e] * wl.E
    masters = [synth.expert_weights(wl, e, device="cuda") for e in range(wl.E)]
    cpu = [m.cpu().numpy() for m in masters]
    pool = wl.E * op.pages_needed(8, wl.H, wl.F)
    ctx = mpe.Context(wl.E, wl.H, wl.F, pool_pages=pool)
    alloc = op.PageAllocator(pool, wl.E, wl.H, wl.F)
    bits0 = oa.allocate_bits(p, W, synth.budget_for(wl, 8.0))
    ctx.quantize_experts(masters, bits0)
    alloc.place(bits0)
    for avg in [7.0, 6.0, 5.0, 4.0, 3.0, 3.75, 4.5, 5.25, 6.0, 6.0]:
        B = synth.budget_for(wl, avg)
        before = alloc.bits.copy()
        old_pages = [list(x) for x in alloc.pages]
        n = ctx.repage(B, p)
        nb = oa.allocate_bits(p, W, B)
        changed = alloc.repage(nb)
        assert n == len(changed)
        assert np.array_equal(ctx.bits(), nb)
        for e in range(wl.E):
            if nb[e] == before[e]:
                assert alloc.pages[e] == old_pages[e]
        _check_expert_state(ctx, wl, nb, cpu, alloc)


def test_pool_exhaustion_is_transactional():
    wl = synth.scaled(synth.WORKLOADS[1], E=4, H=256, F=256)
    p = np.array([0.4, 0.3, 0.2, 0.1])
    masters = [synth.expert_weights(wl, e, device="cuda") for e in range(4)]
    need3 = op.pages_needed(3, wl.H, wl.F)
    pool = 4 * need3 + 1
    ctx = mpe.Context(4, wl.H, wl.F, pool_pages=pool)
    ctx.quantize_experts(masters, np.array([3, 3, 3, 3], np.uint8))
    pte0, pidx0 = ctx.page_table()
    s0 = [ctx.expert_stream(e) for e in range(4)]
    with pytest.raises(mpe.MpeError) as ei:
        ctx.repage(synth.budget_for(wl, 8.0), p)
    assert ei.value.code == -4
    pte1, pidx1 = ctx.page_table()
    assert np.array_equal(pte0, pte1) and np.array_equal(pidx0, pidx1)
    assert all(np.array_equal(a, ctx.expert_stream(e)) for e, a in enumerate(s0))
    assert list(ctx.bits()) == [3, 3, 3, 3]


# ----------------------------------------------------------------------------
# the page's proportional allocator (+ budget repair): a selectable width rule
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("seed", range(8))
def test_allocate_bits_proportional_small(seed):
    rng = np.random.default_rng(100 + seed)
    E = int(rng.integers(1, 40))
    p = rng.dirichlet(np.full(E, 0.5))
    W = [int(x) * 128 for x in rng.integers(1, 50, size=E)]
    B = int(rng.integers(3 * sum(W), 9 * sum(W)))
    got = mpe.allocate_bits_proportional(p, W, B)
    assert np.array_equal(got, oa.allocate_bits_proportional(p, W, B))


@pytest.mark.parametrize("cfg,avg", [(1, 4.5), (2, 4.5), (3, 3.5), (5, 8.0), (5, 6.0), (5, 3.0)])
def test_allocate_bits_proportional_workloads(cfg, avg):
    wl = synth.WORKLOADS[cfg]
    p = synth.importance(wl)
    W = [wl.W_e] * wl.E
    B = synth.budget_for(wl, avg)
    got = mpe.allocate_bits_proportional(p, W, B)
    assert np.array_equal(got, oa.allocate_bits_proportional(p, W, B))
    assert sum(int(b) * w for b, w in zip(got, W)) <= B


def test_allocate_bits_proportional_errors():
    with pytest.raises(mpe.MpeError) as ei:
        mpe.allocate_bits_proportional([1.0, 1.0], [7, 11], 3 * 18 - 1)
    assert ei.value.code == -2
    # all-zero importances: every expert at 3 bits
    assert list(mpe.allocate_bits_proportional([0.0, 0.0, 0.0], [5, 5, 5], 100)) == [3, 3, 3]


def test_repage_with_proportional_allocator():
    wl = synth.scaled(synth.WORKLOADS[1], E=8, H=256, F=256)
    p = synth.importance(wl)
    W = [wl.W_e] * wl.E
    masters = [synth.expert_weights(wl, e, device="cuda") for e in range(wl.E)]
    cpu = [m.cpu().numpy() for m in masters]
    pool = wl.E * op.pages_needed(8, wl.H, wl.F)
    ctx = mpe.Context(wl.E, wl.H, wl.F, pool_pages=pool)
    ctx.set_allocator(mpe.ALLOCATOR_PROPORTIONAL)
    alloc = op.PageAllocator(pool, wl.E, wl.H, wl.F)
    bits0 = oa.allocate_bits_proportional(p, W, synth.budget_for(wl, 8.0))
    ctx.quantize_experts(masters, bits0)
    alloc.place(bits0)
    for avg in [6.0, 4.0, 3.0, 5.0]:
        B = synth.budget_for(wl, avg)
        n = ctx.repage(B, p)
        nb = oa.allocate_bits_proportional(p, W, B)
        assert n == len(alloc.repage(nb))
        assert np.array_equal(ctx.bits(), nb)
        _check_expert_state(ctx, wl, nb, cpu, alloc)
    with pytest.raises(mpe.MpeError):
        ctx.set_allocator(7)
