"""GPU parity for the prefix-compatible variant: codes, layers and the bytes
a width change moves bit-exact against oracle.prefix; the forward pass from
the layered store within the FFN tolerance of the float64 oracle."""
import numpy as np
import pytest
import torch

import synth
from oracle import ffn as of
from oracle import prefix as ox

from _helpers import check_ffn, oracle_moe_parallel

pytestmark = pytest.mark.gpu

mpe = pytest.importorskip("mixed_precision_expert_b200")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixed_precision_expert_b200.build import build
    build()
    assert torch.cuda.is_available()


LAYERS = ("A", "B", "C")


def _check_layers(store, cpu, bits, H, F):
    m = store.absmax()
    for e, w in enumerate(cpu):
        mo, u8 = ox.prefix_codes(w)
        assert m[e] == np.float32(mo)
        n = len(ox.layers_of(int(bits[e])))
        for L in range(3):
            if L < n:
                want = ox.layer_stream(u8, LAYERS[L], H, F).reshape(-1)
                assert np.array_equal(store.read_layer(e, L), want), (e, L)
            else:
                with pytest.raises(mpe.MpeError):
                    store.read_layer(e, L)


def _masters(E, H, F, seed=0, scale=0.02):
    wl = synth.scaled(synth.WORKLOADS[1], E=E, H=H, F=F)
    ms = [synth.expert_weights(wl, e, device="cuda") for e in range(E)]
    if scale != 0.02:
        ms = [(m.float() * (scale / 0.02)).half() for m in ms]
    return wl, ms, [m.cpu().numpy() for m in ms]


def test_quantize_and_repage_schedule():
    E, H, F, P = 4, 256, 384, 4096
    wl, masters, cpu = _masters(E, H, F)
    W_e = 3 * H * F
    n8 = sum(ox.layer_pages(L, H, F, P) for L in LAYERS)
    store = mpe.PrefixStore(E, H, F, page_bytes=P, pool_pages=E * n8)
    pages = ox.LayeredPages(E * n8, E, H, F, P)
    bits = np.array([3, 4, 8, 3], np.uint8)
    store.quantize(masters, bits)
    pages.place(bits)
    _check_layers(store, cpu, bits, H, F)
    for nb in ([8, 8, 8, 8], [3, 4, 8, 3], [4, 3, 3, 8], [3, 3, 3, 3], [8, 4, 3, 4], [8, 4, 3, 4]):
        nb = np.array(nb, np.uint8)
        moved = store.repage(nb)
        enc = pages.repage(nb)
        assert moved == ox.repage_bytes(enc, W_e)
        _check_layers(store, cpu, nb, H, F)
    # lowering widths only moves nothing
    assert store.repage(np.array([3, 4, 3, 3], np.uint8)) == 0


def test_edge_masters_and_pool():
    E, H, F = 3, 128, 128
    wl, masters, cpu = _masters(E, H, F)
    rng = np.random.default_rng(3)
    big = (rng.standard_normal(3 * H * F) * 3000).astype(np.float16)   # large m
    tiny = (rng.integers(-50, 50, size=3 * H * F) * 2.0 ** -24).astype(np.float16)  # subnormal
    zero = np.zeros(3 * H * F, np.float16)
    cpu = [big, tiny, zero]
    masters = [torch.from_numpy(c).cuda() for c in cpu]
    store = mpe.PrefixStore(E, H, F, page_bytes=4096)
    bits = np.array([8, 8, 8], np.uint8)
    store.quantize(masters, bits)
    _check_layers(store, cpu, bits, H, F)
    # a pool too small for a raise leaves everything unchanged
    nA = ox.layer_pages("A", H, F, 4096)
    small = mpe.PrefixStore(E, H, F, page_bytes=4096, pool_pages=3 * nA + 1)
    small.quantize(masters, np.array([3, 3, 3], np.uint8))
    with pytest.raises(mpe.MpeError):
        small.repage(np.array([8, 3, 3], np.uint8))
    _check_layers(small, cpu, np.array([3, 3, 3], np.uint8), H, F)


@pytest.mark.parametrize("bits,page_bytes", [((3, 3, 3, 3), 0), ((4, 4, 4, 4), 0),
                                             ((8, 8, 8, 8), 0), ((3, 4, 8, 4), 0),
                                             ((8, 4, 3, 8), 4096)])
def test_ffn_matches_oracle(bits, page_bytes):
    # 4 KiB pages split a share's run of every layer at page boundaries
    E, H, F = 4, 256, 384
    wl, masters, cpu = _masters(E, H, F, seed=1)
    store = mpe.PrefixStore(E, H, F, page_bytes=page_bytes)
    store.quantize(masters, np.array(bits, np.uint8))
    wl = synth.scaled(synth.WORKLOADS[1], E=E, H=H, F=F, T=40, k=2)
    ids, w = synth.routing(wl, seed=21)
    ids[3, 1] = E + 5  # an invalid id contributes nothing
    x = synth.activations(wl, seed=21)
    got = store.moe_ffn(x.cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    mats = {e: ox.expert_mats(cpu[e], H, F, bits[e]) for e in range(E)}
    ref = of.moe_ffn(x.double().numpy(), ids, w, lambda e: mats[e], E)
    check_ffn(got.double().cpu().numpy(), ref)


def test_ffn_full_size_every_token():
    # the fine-grained layer at full size and its widths, every token; then
    # after a width change that adds and drops layers
    wl = synth.WORKLOADS[3]
    masters = [synth.expert_weights(wl, e, device="cuda") for e in range(wl.E)]
    bits = mpe.allocate_bits(synth.importance(wl), [wl.W_e] * wl.E, wl.budget_bits)
    store = mpe.PrefixStore(wl.E, wl.H, wl.F)
    store.quantize(masters, bits)
    ids, w = synth.routing(wl, seed=5)
    x = synth.activations(wl, seed=5)
    # device reads here, in the main thread; the oracle threads use host copies
    cpu = {int(e): masters[int(e)].cpu().numpy() for e in np.unique(ids) if 0 <= e < wl.E}

    def check(b):
        got = store.moe_ffn(x.cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda())
        torch.cuda.synchronize()
        mats = {}

        def mats_of(e):
            if e not in mats:
                mats[e] = ox.expert_mats(cpu[e], wl.H, wl.F, int(b[e]))
            return mats[e]

        ref = oracle_moe_parallel(x, ids, w, mats_of, wl.E)
        check_ffn(got.double().cpu().numpy(), ref)

    check(bits)
    nb = bits.copy()
    nb[::3] = 8
    nb[1::3] = 3
    store.repage(nb)
    check(nb)
