"""Dynamic repaging at full size (PagedWeight, "Implementation Details": the bit
widths follow the budget as KV-cache occupancy changes): 256 experts, hidden
7168, ffn 2048, 22.5 GB of fp16 masters; quantize at 8 bits average, then the
seeded schedule of 10 decode batches (128 tokens, top-8) alternating with 10
budget changes (average bits 7, 6, 5, 4, 3, 3.75, 4.5, 5.25, 6, 6).

Against the oracle:
* every step: the bit widths (exact program) and the whole page table
  (lowest-free-first allocator);
* the packed codes, absmax and scale of EVERY expert after the initial
  quantize and after the 8 -> 3 sweep ends (the repage to 3 bits average,
  where most experts change), and of 16 seeded changed experts (all of them
  when fewer changed) after every other repage;
* the FFN output of every token on the first decode batch (8 bits) and on the
  batch after the 3-bit repage, and of 16 seeded tokens on every other batch.
The oracle evaluates each expert by value (tests/_helpers.py), which the CPU
tests prove identical to its direct evaluation."""
import numpy as np
import pytest
import torch

import synth
from oracle import allocate as oa
from oracle import pages as op

from _helpers import (OracleExpertByValue, check_experts_in_full, check_ffn, check_page_table,
                      oracle_moe_parallel, workload_masters_gpu)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

mpe = pytest.importorskip("mixed_precision_expert_b200")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixed_precision_expert_b200.build import build
    build()
    assert torch.cuda.is_available()


def test_repage_schedule_full_size():
    wl = synth.WORKLOADS[5]
    E, H, F = wl.E, wl.H, wl.F
    W = [wl.W_e] * E
    p = synth.importance(wl)
    masters = workload_masters_gpu(wl)
    pool = E * op.pages_needed(8, H, F)
    ctx = mpe.Context(E, H, F, pool_pages=pool)
    alloc = op.PageAllocator(pool, E, H, F)
    rng = np.random.default_rng(5005)

    bits = oa.allocate_bits(p, W, synth.budget_for(wl, wl.avg_bits))
    assert np.array_equal(mpe.allocate_bits(p, W, synth.budget_for(wl, wl.avg_bits)), bits)
    ctx.quantize_experts(masters, bits)
    alloc.place(bits)
    check_page_table(ctx, alloc, bits)
    assert check_experts_in_full(ctx, masters, bits, H, F) == E
    assert ctx.status() == 0

    full_ffn_steps, sampled_ffn_steps, full_code_checks = 0, 0, 1
    after_3bit = False
    for i, (kind, arg) in enumerate(synth.schedule(wl)):
        if kind == "decode":
            ids, w = synth.routing(wl, seed=arg)
            x = synth.activations(wl, seed=arg)
            out = ctx.moe_ffn(x.cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda())
            torch.cuda.synchronize()
            assert not (ctx.status() & mpe.STATUS_WAIT_TIMEOUT)
            cur = ctx.bits()

            def mats_of(e, cur=cur):
                return OracleExpertByValue(masters[e].cpu().numpy(), H, F, int(cur[e])).mats()

            got = out.double().cpu().numpy()
            if i == 0 or after_3bit:
                check_ffn(got, oracle_moe_parallel(x, ids, w, mats_of, E))
                full_ffn_steps += 1
                after_3bit = False
            else:
                tok = np.sort(rng.choice(wl.T, 16, replace=False))
                check_ffn(got[tok], oracle_moe_parallel(x, ids, w, mats_of, E, tokens=tok))
                sampled_ffn_steps += 1
        else:
            B = synth.budget_for(wl, arg)
            before = alloc.bits.copy()
            n = ctx.repage(B, p)
            nb = oa.allocate_bits(p, W, B)
            changed = alloc.repage(nb)
            assert n == len(changed)
            assert np.array_equal(ctx.bits(), nb)
            check_page_table(ctx, alloc, nb)
            assert all(nb[e] != before[e] for e in changed)
            if arg == 3.0 and not after_3bit and full_code_checks == 1:
                # the end of the 8 -> 3 sweep: every expert, changed or not
                assert check_experts_in_full(ctx, masters, nb, H, F) == E
                full_code_checks += 1
                after_3bit = True
            elif changed:
                pick = changed if len(changed) <= 16 else \
                    sorted(rng.choice(changed, 16, replace=False).tolist())
                assert check_experts_in_full(ctx, masters, nb, H, F, experts=pick) == len(pick)
            assert ctx.status() == 0
    assert full_code_checks == 2
    assert full_ffn_steps == 2 and sampled_ffn_steps == 8
    ctx.close()
