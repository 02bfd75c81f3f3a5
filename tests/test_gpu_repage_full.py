"""Dynamic repaging at full size (PagedWeight, "Implementation Details": the bit
widths follow the budget as KV-cache occupancy changes): 256 experts, hidden
7168, ffn 2048, 22.5 GB of fp16 masters; quantize at 8 bits average, then the
seeded schedule of 10 decode batches (128 tokens, top-8) alternating with 10
budget changes (average bits 7, 6, 5, 4, 3, 3.75, 4.5, 5.25, 6, 6).

Against the oracle at every step: the bit widths (exact DP) and the whole page
table (lowest-free-first allocator). On samples, because the float64 oracle
takes seconds per expert at this size: the packed codes of seeded experts after
the initial quantize and after repages (every changed expert's width is then
pinned by the page-table check), and the FFN output of one seeded token on
three decode steps, including the all-3-bit state."""
import numpy as np
import pytest
import torch

import synth
from oracle import allocate as oa
from oracle import pages as op

from _helpers import OracleExpert, check_ffn, oracle_moe

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

mpe = pytest.importorskip("mixed_precision_expert_b200")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixed_precision_expert_b200.build import build
    build()
    assert torch.cuda.is_available()


def _master_cpu(wl, e):
    return synth.expert_weights(wl, e).numpy()


def _check_table(ctx, alloc, bits):
    pte, pidx = ctx.page_table()
    table = alloc.table()
    assert np.array_equal(pte["bits"], np.asarray(bits, np.uint8))
    assert np.array_equal(pte["first"], table.first)
    assert np.array_equal(pte["n_pages"], table.n_pages)
    assert np.array_equal(pidx, table.page_idx)


def _check_codes(ctx, wl, e, b):
    ref = OracleExpert(_master_cpu(wl, e), wl.H, wl.F, int(b))
    assert np.array_equal(ctx.expert_stream(e), ref.stream()), f"expert {e} at {b} bits"
    s, m = ctx.scales()
    assert s[e] == ref.s and m[e] == np.float32(ref.m)


def test_repage_schedule_full_size():
    wl = synth.WORKLOADS[5]
    E, H, F = wl.E, wl.H, wl.F
    W = [wl.W_e] * E
    p = synth.importance(wl)
    masters = []
    for e in range(E):
        t = torch.empty(wl.W_e, dtype=torch.float16, device="cuda")
        synth.fill_expert_weights(wl, e, t)
        masters.append(t)
    pool = E * op.pages_needed(8, H, F)
    ctx = mpe.Context(E, H, F, pool_pages=pool)
    alloc = op.PageAllocator(pool, E, H, F)
    rng = np.random.default_rng(5005)

    bits = oa.allocate_bits(p, W, synth.budget_for(wl, wl.avg_bits))
    assert np.array_equal(mpe.allocate_bits(p, W, synth.budget_for(wl, wl.avg_bits)), bits)
    ctx.quantize_experts(masters, bits)
    alloc.place(bits)
    _check_table(ctx, alloc, bits)
    for e in rng.choice(E, 2, replace=False):
        _check_codes(ctx, wl, int(e), bits[e])
    assert ctx.status() == 0

    checked_ffn = 0
    for i, (kind, arg) in enumerate(synth.schedule(wl)):
        if kind == "decode":
            ids, w = synth.routing(wl, seed=arg)
            x = synth.activations(wl, seed=arg)
            out = ctx.moe_ffn(x.cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda())
            torch.cuda.synchronize()
            assert not (ctx.status() & mpe.STATUS_WAIT_TIMEOUT)
            # the first batch (8 bits), the batch after the 8 -> 3 sweep ends
            # (all 3-bit) and the last batch
            if i in (0, 10, 18):
                tok = np.array([int(rng.integers(0, wl.T))])
                cur = ctx.bits()

                def mats_of(e, cur=cur):
                    return OracleExpert(_master_cpu(wl, e), H, F, int(cur[e])).mats()

                got = out.double().cpu().numpy()[tok]
                check_ffn(got, oracle_moe(x, ids, w, mats_of, E, tokens=tok))
                checked_ffn += 1
        else:
            B = synth.budget_for(wl, arg)
            before = alloc.bits.copy()
            n = ctx.repage(B, p)
            nb = oa.allocate_bits(p, W, B)
            changed = alloc.repage(nb)
            assert n == len(changed)
            assert np.array_equal(ctx.bits(), nb)
            _check_table(ctx, alloc, nb)
            if changed:
                e = int(rng.choice(changed))
                assert nb[e] != before[e]
                _check_codes(ctx, wl, e, nb[e])
            assert ctx.status() == 0
    assert checked_ffn == 3
    ctx.close()
