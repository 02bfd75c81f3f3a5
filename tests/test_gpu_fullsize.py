"""Full-size GPU parity on the decode workloads (PagedWeight, "Implementation
Details": the per-expert absmax quantizer; "Dynamic Paging": pages of 8/4/3
bits addressed through a page table keyed by expert ID, fetched and
dequantized on the fly by the expert FFN).

Mixtral-shaped layer (8 experts, hidden 4096, ffn 14336, 0.1 % outliers at
10 sigma, 16 tokens top-2, 4.5 bits average) and the fine-grained layer (128
experts, hidden 2048, ffn 768, 64 tokens top-8 with Zipf skew, 3.5 bits
average): bit-exact widths, absmax, scales, page table and the WHOLE packed
stream of every expert; the FFN output of every token within the tolerance.
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


def _quantized_layer(wl):
    masters = workload_masters_gpu(wl)
    p = synth.importance(wl)
    W = [wl.W_e] * wl.E
    bits = oa.allocate_bits(p, W, wl.budget_bits, state_cap=mpe.ALLOC_STATE_CAP)
    assert np.array_equal(mpe.allocate_bits(p, W, wl.budget_bits), bits)
    ctx = mpe.Context(wl.E, wl.H, wl.F)
    ctx.quantize_experts(masters, bits)
    alloc = op.PageAllocator(wl.E * op.pages_needed(8, wl.H, wl.F), wl.E, wl.H, wl.F)
    alloc.place(bits)
    return ctx, masters, bits, alloc


def _forward(ctx, x, ids, w):
    out = ctx.moe_ffn(x.cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    assert not (ctx.status() & mpe.STATUS_WAIT_TIMEOUT)
    return out.double().cpu().numpy()


def _mats_of(masters, bits, wl):
    def mats(e):
        return OracleExpertByValue(masters[e].cpu().numpy(), wl.H, wl.F, int(bits[e])).mats()
    return mats


def test_mixtral_decode_layer_full_size():
    wl = synth.WORKLOADS[2]
    ctx, masters, bits, alloc = _quantized_layer(wl)
    check_page_table(ctx, alloc, bits)
    assert check_experts_in_full(ctx, masters, bits, wl.H, wl.F) == wl.E
    # every expert's absmax is one of the 10-sigma outliers
    _, absmax = ctx.scales()
    assert np.all(absmax == np.float32(np.float16(wl.outlier_value)))
    assert ctx.status() == 0
    ids, w = synth.routing(wl)
    x = synth.activations(wl)
    got = _forward(ctx, x, ids, w)
    ref = oracle_moe_parallel(x, ids, w, _mats_of(masters, bits, wl), wl.E, workers=4)
    check_ffn(got, ref)
    assert ctx.status() == 0
    ctx.close()


def test_finegrained_decode_layer_full_size():
    wl = synth.WORKLOADS[3]
    ctx, masters, bits, alloc = _quantized_layer(wl)
    assert set(np.unique(bits).tolist()) >= {3, 4}
    check_page_table(ctx, alloc, bits)
    assert check_experts_in_full(ctx, masters, bits, wl.H, wl.F) == wl.E
    ids, w = synth.routing(wl)
    x = synth.activations(wl)
    got = _forward(ctx, x, ids, w)
    check_ffn(got, oracle_moe_parallel(x, ids, w, _mats_of(masters, bits, wl), wl.E))
    assert ctx.status() == 0
    ctx.close()
