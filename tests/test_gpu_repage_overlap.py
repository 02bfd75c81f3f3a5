"""GPU parity of the overlapped repage (mpe_repage_async / mpe_repage_commit):
the budget change of PagedWeight's scheduler ("Implementation Details": page
sizes follow KV-cache occupancy) while forward passes go on. Before the commit
a forward pass reads the old pages (the old widths' layer); after it the
widths, page table, scales, packed codes and the layer match the oracle's
overlapped page rule (new pages from the free pool, old pages freed at the
commit), bit-exactly except the FFN (rel-Frobenius / max-abs tolerance)."""
import numpy as np
import pytest
import torch

import synth
from oracle import allocate as oa
from oracle import pages as op

from _helpers import OracleExpert, check_ffn, oracle_moe

pytestmark = pytest.mark.gpu

mpe = pytest.importorskip("mixed_precision_expert_b200")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixed_precision_expert_b200.build import build
    build()
    assert torch.cuda.is_available()


def _state_matches(ctx, wl, bits, cpu, alloc):
    scales, absmax = ctx.scales()
    pte, pidx = ctx.page_table()
    table = alloc.table()
    assert np.array_equal(pte["bits"], np.asarray(bits, np.uint8))
    assert np.array_equal(pte["first"], table.first)
    assert np.array_equal(pte["n_pages"], table.n_pages)
    assert np.array_equal(pidx, table.page_idx)
    for e in range(wl.E):
        ox = OracleExpert(cpu[e], wl.H, wl.F, int(bits[e]))
        assert scales[e] == ox.s and absmax[e] == np.float32(ox.m)
        assert np.array_equal(ctx.expert_stream(e), ox.stream()), e


def _layer_ref(wl, bits, cpu, x, ids, w):
    ox = [OracleExpert(cpu[e], wl.H, wl.F, int(b)) for e, b in enumerate(bits)]
    return oracle_moe(x, ids, w, lambda e: ox[e].mats(), wl.E)


def test_overlapped_repage_serves_old_pages_until_commit():
    wl = synth.scaled(synth.WORKLOADS[1], E=8, H=256, F=512)
    p = synth.importance(wl)
    W = [wl.W_e] * wl.E
    masters = [synth.expert_weights(wl, e, device="cuda") for e in range(wl.E)]
    cpu = [m.cpu().numpy() for m in masters]
    need8 = op.pages_needed(8, wl.H, wl.F)
    pool = wl.E * need8 + wl.E * need8 // 2
    ctx = mpe.Context(wl.E, wl.H, wl.F, pool_pages=pool)
    alloc = op.PageAllocator(pool, wl.E, wl.H, wl.F)
    bits = oa.allocate_bits(p, W, synth.budget_for(wl, 8.0))
    ctx.quantize_experts(masters, bits)
    alloc.place(bits)
    ids, w = synth.routing(wl, seed=11)
    x = synth.activations(wl, seed=11)
    xg, idg, wg = x.cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda()
    for avg in [6.0, 4.0, 3.0, 5.0, 5.0]:
        old_bits = alloc.bits.copy()
        B = synth.budget_for(wl, avg)
        n = ctx.repage_async(B, p)
        nb = oa.allocate_bits(p, W, B)
        changed = alloc.repage_overlapped(nb)
        assert n == len(changed)
        assert np.array_equal(ctx.bits(), nb)  # the new widths, before the commit
        # forward passes before the commit: the old pages, i.e. the old widths
        out = ctx.moe_ffn(xg, idg, wg)
        torch.cuda.synchronize()
        check_ffn(out.double().cpu().numpy(), _layer_ref(wl, old_bits, cpu, x, ids, w))
        with pytest.raises(mpe.MpeError) as ei:  # one pending at a time
            ctx.repage_async(B, p)
        assert ei.value.code == -6
        assert ctx.repage_commit(wait=True)
        alloc.commit()
        _state_matches(ctx, wl, nb, cpu, alloc)
        out = ctx.moe_ffn(xg, idg, wg)
        torch.cuda.synchronize()
        check_ffn(out.double().cpu().numpy(), _layer_ref(wl, nb, cpu, x, ids, w))
    assert ctx.repage_commit(wait=False)  # nothing pending
    assert ctx.status() == 0


def test_overlapped_repage_needs_free_pages():
    wl = synth.scaled(synth.WORKLOADS[1], E=4, H=256, F=256)
    p = np.array([0.4, 0.3, 0.2, 0.1])
    masters = [synth.expert_weights(wl, e, device="cuda") for e in range(4)]
    pool = 4 * op.pages_needed(8, wl.H, wl.F)  # no room beside the 8-bit pages
    ctx = mpe.Context(4, wl.H, wl.F, pool_pages=pool)
    ctx.quantize_experts(masters, np.array([8, 8, 8, 8], np.uint8))
    pte0, pidx0 = ctx.page_table()
    with pytest.raises(mpe.MpeError) as ei:
        ctx.repage_async(synth.budget_for(wl, 4.0), p)
    assert ei.value.code == -4
    pte1, pidx1 = ctx.page_table()
    assert np.array_equal(pte0, pte1) and np.array_equal(pidx0, pidx1)
    assert list(ctx.bits()) == [8, 8, 8, 8]
    # the synchronous repage still works (it frees before it allocates)
    assert ctx.repage(synth.budget_for(wl, 4.0), p) > 0


def test_commit_without_wait_and_sync_repage_after_async():
    wl = synth.scaled(synth.WORKLOADS[1], E=4, H=256, F=256)
    p = synth.importance(wl)[:4] / synth.importance(wl)[:4].sum()
    W = [wl.W_e] * 4
    masters = [synth.expert_weights(wl, e, device="cuda") for e in range(4)]
    cpu = [m.cpu().numpy() for m in masters]
    need8 = op.pages_needed(8, wl.H, wl.F)
    pool = 8 * need8
    ctx = mpe.Context(4, wl.H, wl.F, pool_pages=pool)
    alloc = op.PageAllocator(pool, 4, wl.H, wl.F)
    ctx.quantize_experts(masters, np.array([8, 8, 8, 8], np.uint8))
    alloc.place(np.array([8, 8, 8, 8], np.uint8))
    B = synth.budget_for(wl, 4.0)
    ctx.repage_async(B, p)
    alloc.repage_overlapped(oa.allocate_bits(p, W, B))
    torch.cuda.synchronize()
    # the device work is done: a non-waiting commit switches
    assert ctx.repage_commit(wait=False)
    alloc.commit()
    _state_matches(ctx, wl, alloc.bits, cpu, alloc)
    # an overlapped repage left pending is committed by a synchronous one
    B2 = synth.budget_for(wl, 3.0)
    ctx.repage_async(synth.budget_for(wl, 6.0), p)
    alloc.repage_overlapped(oa.allocate_bits(p, W, synth.budget_for(wl, 6.0)))
    ctx.repage(B2, p)
    alloc.commit()
    alloc.repage(oa.allocate_bits(p, W, B2))
    _state_matches(ctx, wl, alloc.bits, cpu, alloc)
