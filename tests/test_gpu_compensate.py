"""GPU parity for salient-channel error compensation (DecDEC summary, 3.1-3.2
and Figure 4): the channel choice bit-exact against the oracle, the
compensated layer within the FFN tolerance of the float64 oracle, and its two
ends -- every channel kept gives the fp16-weight layer."""
import numpy as np
import pytest
import torch

import synth
from oracle import compensate as oc
from oracle import ffn as of
from oracle import route as orr

from _helpers import OracleExpert, check_ffn

pytestmark = pytest.mark.gpu

mpe = pytest.importorskip("mixed_precision_expert_b200")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixed_precision_expert_b200.build import build
    build()
    assert torch.cuda.is_available()


@pytest.mark.parametrize("rows,cols,seed", [(37, 300, 0), (5, 4096, 1), (64, 7, 2), (3, 14336, 3)])
def test_select_salient_matches_oracle(rows, cols, seed):
    rng = np.random.default_rng(seed)
    # few distinct magnitudes (many ties), both signs, zeros of both signs
    vals = rng.choice([0.0, -0.0, 0.5, -0.5, 1.5, -2.0, 3.0, 1e-30, -7.0], size=(rows, cols))
    vals[:, rng.integers(0, cols, size=max(1, cols // 50))] *= 40.0
    x = torch.from_numpy(vals).to(torch.bfloat16).cuda()
    xf = x.double().cpu().numpy()
    for n in (1, 2, 5, 64, 256):
        got = mpe.select_salient(x, n).cpu().numpy()
        for r in range(rows):
            want = oc.salient_channels(xf[r], n)
            m = min(n, cols)
            assert np.array_equal(got[r, :m], want), (n, r)


def _layer(E, H, F, bits, seed=0, outliers=True, T=16, k=2):
    wl = synth.scaled(synth.WORKLOADS[1], E=E, H=H, F=F, T=T, k=k)
    masters = [synth.expert_weights(wl, e, device="cuda") for e in range(E)]
    ctx = mpe.Context(E, H, F, path=mpe.PATH_DECODE)
    ctx.quantize_experts(masters, np.asarray(bits, np.uint8))
    cpu = [m.cpu().numpy() for m in masters]

    def split(a):
        return (a[:F * H].reshape(F, H), a[F * H:2 * F * H].reshape(F, H),
                a[2 * F * H:].reshape(H, F))

    hats = {e: OracleExpert(cpu[e], H, F, int(bits[e])).mats() for e in range(E)}
    fp16 = {e: split(cpu[e].astype(np.float64)) for e in range(E)}
    ids, w = synth.routing(wl, seed=100 + seed)
    x = synth.activations(wl, seed=100 + seed)
    if outliers:
        rng = np.random.default_rng(seed)
        xx = x.float()
        xx[:, torch.from_numpy(rng.choice(H, max(2, H // 64), replace=False))] *= 30.0
        x = xx.to(torch.bfloat16)
    return ctx, x, ids, w, hats, fp16


# The device ranks h after rounding it to bf16 (a relative error of at most
# 2^-8 each, round to nearest with 8 significant bits), from g and v
# accumulated in fp32 and a silu with a fast divide: that part is far below
# the rounding, bounded here by 1e-5 of the row's largest |h| per value
# (tolerance 2 * 1e-5 for the pair). A left-out channel may then exceed a
# kept one only by the two roundings and the two pre-rounding errors.
BF16_REL = 2.0 ** -8
H_ERR_ABS = 2e-5


def _oracle_with_device_masks(ctx, x, ids, w, hats, fp16, E, H, F, n):
    """Oracle output under the device's down-projection masks, after checking
    that the device's x masks are the oracle's (exact inputs: a unique answer)
    and that each h mask is a valid choice on the oracle's h (the device chose
    on bf16 h from fp32 arithmetic, so near-ties may fall either way)."""
    T, k = ids.shape
    xd = x.double().numpy()
    sel_x = ctx.kept_channels(0, T, n)
    sel_h = ctx.kept_channels(1, T * k, n)
    for t in range(T):
        assert np.array_equal(sel_x[t, :min(n, H)], oc.salient_channels(xd[t], n)), t
    _, _, inv = orr.route(ids, E)
    masks = {}
    for t in range(T):
        for j in range(k):
            pos = int(inv[t * k + j])
            if pos < 0:
                continue
            e = int(ids[t, j])
            w1h, w3h, _ = hats[e]
            w1, w3, _ = fp16[e]
            h = of.silu(oc.compensated_linear(w1h, w1, xd[t], n)) * \
                oc.compensated_linear(w3h, w3, xd[t], n)
            m = sel_h[pos, :min(n, F)]
            assert oc.is_valid_choice(h, m, n, H_ERR_ABS * np.abs(h).max(), rel=BF16_REL), (t, j)
            masks[(t, j)] = m
    return oc.moe_ffn_compensated(xd, ids, w, lambda e: hats[e], lambda e: fp16[e], E, n,
                                  down_masks=masks)


def _run(ctx, x, ids, w):
    out = ctx.moe_ffn(x.cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    assert not (ctx.status() & mpe.STATUS_WAIT_TIMEOUT)
    return out.double().cpu().numpy()


@pytest.mark.parametrize("n", [8, 64])
@pytest.mark.parametrize("bits", [(3, 4, 8, 3), (3, 3, 3, 3)])
def test_compensated_layer_matches_oracle(n, bits):
    E, H, F = 4, 512, 384
    ctx, x, ids, w, hats, fp16 = _layer(E, H, F, bits, seed=n)
    plain = _run(ctx, x, ids, w)
    ctx.set_compensation(n)
    got = _run(ctx, x, ids, w)
    xd = x.double().numpy()
    check_ffn(got, _oracle_with_device_masks(ctx, x, ids, w, hats, fp16, E, H, F, n))
    # closer to the fp16-weight layer than without compensation
    full = of.moe_ffn(xd, ids, w, lambda e: fp16[e], E)
    assert np.linalg.norm(got - full) < np.linalg.norm(plain - full)
    # switching off gives the plain path back, bit for bit
    ctx.set_compensation(0)
    assert np.array_equal(_run(ctx, x, ids, w), plain)
    assert ctx.status() == 0


def test_every_channel_gives_the_fp16_layer():
    E, H, F = 3, 128, 256  # both input widths within the 256-channel cap
    ctx, x, ids, w, hats, fp16 = _layer(E, H, F, (3, 4, 3), seed=5)
    ctx.set_compensation(256)
    got = _run(ctx, x, ids, w)
    xd = x.double().numpy()
    full = of.moe_ffn(xd, ids, w, lambda e: fp16[e], E)
    check_ffn(got, full)
    plain_ref = of.moe_ffn(xd, ids, w, lambda e: hats[e], E)
    assert np.linalg.norm(got - full) < 0.1 * np.linalg.norm(plain_ref - full)


def test_error_falls_with_channels_and_host_store():
    E, H, F = 4, 1024, 512
    ctx, x, ids, w, hats, fp16 = _layer(E, H, F, (3, 3, 4, 3), seed=7)
    xd = x.double().numpy()
    full = of.moe_ffn(xd, ids, w, lambda e: fp16[e], E)
    errs = []
    for n in (0, 4, 16, 64, 256):
        ctx.set_compensation(n)
        errs.append(np.linalg.norm(_run(ctx, x, ids, w) - full))
    assert all(b < a for a, b in zip(errs, errs[1:])), errs
    # the same values from a store in mapped host memory
    ctx.set_compensation(16)
    dev = _run(ctx, x, ids, w)
    ctx.set_compensation(16, mpe.STORE_HOST)
    assert np.array_equal(_run(ctx, x, ids, w), dev)


def test_compensation_follows_repage():
    E, H, F = 4, 256, 256
    wl = synth.scaled(synth.WORKLOADS[1], E=E, H=H, F=F, T=16, k=2)
    ctx, x, ids, w, hats, fp16 = _layer(E, H, F, (8, 8, 8, 8), seed=9)
    ctx.set_compensation(32)
    p = synth.importance(wl)
    ctx.repage(synth.budget_for(wl, 3.5), p)
    bits = ctx.bits()
    masters = [fp16[e] for e in range(E)]
    hats2 = {}
    for e in range(E):
        flat = np.concatenate([m.reshape(-1) for m in masters[e]]).astype(np.float16)
        hats2[e] = OracleExpert(flat, H, F, int(bits[e])).mats()
    got = _run(ctx, x, ids, w)
    check_ffn(got, _oracle_with_device_masks(ctx, x, ids, w, hats2, fp16, E, H, F, 32))


def test_compensation_errors():
    E, H, F = 2, 128, 128
    ctx = mpe.Context(E, H, F)
    with pytest.raises(mpe.MpeError):
        ctx.set_compensation(8)  # before quantize
    ctx2, x, ids, w, _, _ = _layer(E, H, F, (4, 4), seed=11)
    with pytest.raises(mpe.MpeError):
        ctx2.set_compensation(257)
    with pytest.raises(mpe.MpeError):
        ctx2.set_compensation(8, 5)
    ctx2.set_compensation(8)
    ctx2.set_path(mpe.PATH_PREFILL)
    with pytest.raises(mpe.MpeError):
        ctx2.moe_ffn(x.cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda())
    ctx2.set_path(mpe.PATH_AUTO)
    _run(ctx2, x, ids, w)
