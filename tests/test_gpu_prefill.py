"""GPU parity of the tensor-core (prefill) expert FFN path against the float64
dequantize-then-multiply oracle (PagedWeight, "Dynamic Paging"; tolerance
rel-Frobenius <= 5e-3, max-abs <= 2e-2 * max|oracle|).

The path is forced with MPE_PATH_PREFILL so that small layers, single tokens and
ragged 192-token work groups all run through it; the full-size case is the
fine-grained layer (128 experts, hidden 2048, ffn 768) with 8192 tokens top-8,
checked on every token."""
import numpy as np
import pytest
import torch

import synth

from _helpers import check_ffn, oracle_moe, oracle_moe_parallel
from test_gpu_route_ffn import _layer, _run

pytestmark = pytest.mark.gpu

mpe = pytest.importorskip("mixed_precision_expert_b200")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixed_precision_expert_b200.build import build
    build()
    assert torch.cuda.is_available()


def test_prefill_odd_tile_count_and_group_boundaries():
    # hidden 384: the down projection has 3 output tiles of 128, so its last
    # tile pair has one tile; ~330 assignments per expert split into a full
    # 192-token group and a ragged one
    wl = synth.scaled(synth.WORKLOADS[1], E=3, H=384, F=256, T=500, k=2)
    ctx, _, mats_of = _layer(wl, np.array([3, 8, 4], np.uint8), path=mpe.PATH_PREFILL)
    ids, w = synth.routing(wl)
    assert np.bincount(ids.ravel(), minlength=3).max() > 192
    x = synth.activations(wl)
    check_ffn(_run(ctx, x, ids, w), oracle_moe(x, ids, w, mats_of, wl.E))
    assert ctx.status() == 0


@pytest.mark.parametrize("bits", [(3,) * 4, (4,) * 4, (8,) * 4, (3, 4, 8, 3)])
def test_prefill_each_width(bits):
    # ~150 assignments per expert: one ragged group of up to 192 tokens each;
    # 4 K-steps per tile and 2 feature tiles in both contractions
    wl = synth.scaled(synth.WORKLOADS[1], E=4, H=256, F=256, T=300, k=2)
    ctx, _, mats_of = _layer(wl, np.array(bits, np.uint8), path=mpe.PATH_PREFILL)
    ids, w = synth.routing(wl)
    x = synth.activations(wl)
    check_ffn(_run(ctx, x, ids, w), oracle_moe(x, ids, w, mats_of, wl.E))
    assert ctx.status() == 0


def test_prefill_edge_token_counts():
    wl = synth.scaled(synth.WORKLOADS[1], E=6, H=384, F=128, T=400, k=3)
    ctx, _, mats_of = _layer(wl, np.array([3, 4, 8, 4, 3, 8], np.uint8),
                             path=mpe.PATH_PREFILL)
    x = synth.activations(wl)
    rng = np.random.default_rng(11)
    cases = []
    # one token
    cases.append((x[:1], np.array([[2, 0, 5]], np.int32)))
    # every token on expert 1 (four work groups, the last ragged), expert 4 unused
    ids = np.stack([np.ones(400, np.int32), rng.integers(0, 4, 400).astype(np.int32),
                    np.full(400, 5, np.int32)], 1)
    cases.append((x, ids))
    # exactly one full group on expert 0 and a 1-token group on expert 3
    ids = np.zeros((129, 1), np.int32)
    ids[128, 0] = 3
    cases.append((x[:129], ids))
    # 127 tokens spread over all experts
    cases.append((x[:127], rng.integers(0, 6, size=(127, 3)).astype(np.int32)))
    for xi, ids in cases:
        w = rng.random(ids.shape).astype(np.float32)
        check_ffn(_run(ctx, xi.contiguous(), ids, w), oracle_moe(xi, ids, w, mats_of, wl.E))
    assert ctx.status() == 0


def test_prefill_invalid_ids_are_dropped():
    wl = synth.scaled(synth.WORKLOADS[1], E=4, H=128, F=256, T=200, k=2)
    ctx, _, mats_of = _layer(wl, np.array([4, 4, 8, 3], np.uint8), path=mpe.PATH_PREFILL)
    x = synth.activations(wl)
    ids, w = synth.routing(wl)
    ids[::7, 1] = 9
    ids[3, 0] = -1
    got = _run(ctx, x, ids, w)
    assert ctx.status(clear=True) & mpe.STATUS_BAD_EXPERT_ID
    check_ffn(got, oracle_moe(x, ids, w, mats_of, wl.E))


def test_prefill_small_pages():
    # 4 KiB pages hold 5 / 4 / 2 chunks of width 3 / 4 / 8, so each row's page
    # cursor crosses pages inside a tile
    wl = synth.scaled(synth.WORKLOADS[1], E=3, H=512, F=384, T=200, k=2)
    bits = np.array([3, 4, 8], np.uint8)
    masters = [synth.expert_weights(wl, e, device="cuda") for e in range(wl.E)]
    ctx = mpe.Context(wl.E, wl.H, wl.F, page_bytes=4096, path=mpe.PATH_PREFILL)
    ctx.quantize_experts(masters, bits)
    _, _, mats_of = _layer(wl, bits, path=mpe.PATH_PREFILL)
    ids, w = synth.routing(wl)
    x = synth.activations(wl)
    check_ffn(_run(ctx, x, ids, w), oracle_moe(x, ids, w, mats_of, wl.E))


def test_prefill_matches_decode_path_on_same_layer():
    wl = synth.scaled(synth.WORKLOADS[1], E=8, H=256, F=512, T=256, k=2)
    ctx, _, mats_of = _layer(wl)
    ids, w = synth.routing(wl)
    x = synth.activations(wl)
    ref = oracle_moe(x, ids, w, mats_of, wl.E)
    ctx.set_path(mpe.PATH_DECODE)
    dec = _run(ctx, x, ids, w)
    ctx.set_path(mpe.PATH_PREFILL)
    pre = _run(ctx, x, ids, w)
    check_ffn(dec, ref)
    check_ffn(pre, ref)
    # both paths accumulate in fp32 and round h and the output to bf16: they
    # agree far inside the oracle tolerance
    assert np.linalg.norm(pre - dec) / np.linalg.norm(ref) < 5e-3


def test_prefill_finegrained_full_size():
    # 128 experts, hidden 2048, ffn 768, 8192 tokens top-8 with Zipf-skewed
    # routing, 3.5 bits average; the automatic path choice takes the tensor cores
    wl = synth.WORKLOADS[4]
    ctx, _, mats_of = _layer(wl)
    ids, w = synth.routing(wl)
    x = synth.activations(wl)
    ctx.profile(True)
    got = _run(ctx, x, ids, w)
    prof = ctx.profile_read()
    ctx.profile(False)
    assert prof["tc_gate_up"][1] == 1 and prof["tc_down"][1] == 1
    assert prof["gate_up"][1] == 0 and prof["down"][1] == 0
    # every token: each heavy expert's 192-token work groups, ragged tails and
    # the experts with a handful of tokens
    check_ffn(got, oracle_moe_parallel(x, ids, w, mats_of, wl.E))
    assert ctx.status() == 0
