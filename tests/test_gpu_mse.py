"""GPU parity for the measured per-expert loss and the loss-table allocator
(PagedWeight, "Quality-Aware Quantization": L(b) is a loss such as the mean
squared error; experts differ in sensitivity): bit-exact against the float64
oracle."""
import numpy as np
import pytest
import torch

import synth
from oracle import allocate as oa
from oracle import pages as op
from oracle import quantize as oq

from _helpers import OracleExpert

pytestmark = pytest.mark.gpu

mpe = pytest.importorskip("mixed_precision_expert_b200")

WIDTHS = (3, 4, 8)


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixed_precision_expert_b200.build import build
    build()
    assert torch.cuda.is_available()


def _oracle_loss(cpu_masters, experts=None):
    experts = range(len(cpu_masters)) if experts is None else experts
    return {e: [oq.quantization_mse(cpu_masters[e], b) for b in WIDTHS] for e in experts}


def _context(wl, masters, bits):
    ctx = mpe.Context(wl.E, wl.H, wl.F)
    ctx.quantize_experts(masters, bits)
    return ctx


def test_measure_loss_tiny_layer():
    wl = synth.WORKLOADS[1]
    masters = [synth.expert_weights(wl, e, device="cuda") for e in range(wl.E)]
    cpu = [m.cpu().numpy() for m in masters]
    ctx = _context(wl, masters, np.full(wl.E, 4, np.uint8))
    got = ctx.measure_loss()
    ref = _oracle_loss(cpu)
    for e in range(wl.E):
        assert list(got[e]) == ref[e], (e, got[e], ref[e])
    # cached: a second call returns the same values
    assert np.array_equal(ctx.measure_loss(), got)


def test_measure_loss_edge_experts():
    # wide scales (s_3 >= 1: 128-bit sums), half-integer quotients, a zero
    # expert, subnormal-only weights, a single outlier, a ragged last segment
    wl = synth.scaled(synth.WORKLOADS[1], E=6, H=128, F=384)
    rng = np.random.default_rng(11)
    n = wl.W_e
    cpu = []
    cpu.append((rng.standard_normal(n) * 40.0).astype(np.float16))                # wide
    m = np.float16(1.5)
    s = np.float32(np.float64(m) / 3)
    half = (rng.integers(-6, 7, size=n) * (np.float64(s) / 2)).astype(np.float16)
    half[0] = m
    cpu.append(half)                                                                # ties
    cpu.append(np.zeros(n, np.float16))                                             # zero
    cpu.append((rng.integers(-1023, 1024, size=n) * 2.0 ** -24).astype(np.float16)) # subnormal
    one = np.zeros(n, np.float16)
    one[n // 2] = np.float16(-3.0e3)
    one[: n // 3] = (rng.standard_normal(n // 3) * 0.5).astype(np.float16)
    cpu.append(one)                                                                 # outlier
    cpu.append((rng.standard_normal(n) * 7000.0).astype(np.float16))              # huge
    for c in cpu:
        assert np.all(np.isfinite(c))
    masters = [torch.from_numpy(c).cuda() for c in cpu]
    ctx = _context(wl, masters, np.full(wl.E, 8, np.uint8))
    got = ctx.measure_loss()
    ref = _oracle_loss(cpu)
    for e in range(wl.E):
        assert list(got[e]) == ref[e], (e, got[e], ref[e])
    assert list(got[2]) == [0.0, 0.0, 0.0]


def test_measure_loss_nonfinite_master():
    wl = synth.scaled(synth.WORKLOADS[1], E=2, H=128, F=128)
    a = torch.zeros(wl.W_e, dtype=torch.float16, device="cuda")
    b = a.clone()
    b[17] = float("inf")
    ctx = _context(wl, [a, b], np.full(2, 4, np.uint8))
    got = ctx.measure_loss()
    assert list(got[0]) == [0.0, 0.0, 0.0]
    assert np.isnan(got[1]).all()


def test_measure_loss_full_size_sampled():
    # the fine-grained layer (128 experts, H 2048, F 768) at full size; the
    # oracle checks two sampled experts
    wl = synth.WORKLOADS[3]
    masters = [synth.expert_weights(wl, e, device="cuda") for e in range(wl.E)]
    ctx = _context(wl, masters, np.full(wl.E, 3, np.uint8))
    got = ctx.measure_loss()
    for e in (0, 77):
        ref = [oq.quantization_mse(masters[e].cpu().numpy(), b) for b in WIDTHS]
        assert list(got[e]) == ref, (e, got[e], ref)
    assert np.all(got[:, 0] > got[:, 1]) and np.all(got[:, 1] > got[:, 2])


@pytest.mark.parametrize("seed", range(12))
def test_allocate_bits_table_small(seed):
    rng = np.random.default_rng(300 + seed)
    E = int(rng.integers(1, 40))
    p = rng.dirichlet(np.full(E, 0.6))
    if seed % 4 == 0:
        p[rng.integers(0, E)] = 0.0
    L = rng.uniform(1e-7, 1e-2, size=(E, 3))
    if seed % 3:
        L = np.sort(L, axis=1)[:, ::-1].copy()  # decreasing in b, like measured losses
    W = [int(x) for x in rng.choice([2048, 4096, 6144], size=E)] if seed % 2 else [393216] * E
    sw = sum(W)
    for B in (3 * sw, int(rng.integers(3 * sw, 8 * sw)), 8 * sw, 9 * sw):
        got = mpe.allocate_bits_table(p, L, W, B)
        ref = oa.allocate_bits_table(p, L, W, B)
        assert np.array_equal(got, ref), (B, got, ref)


def test_allocate_bits_table_errors():
    p = np.full(4, 0.25)
    L = np.full((4, 3), 1e-3)
    with pytest.raises(mpe.MpeError):
        mpe.allocate_bits_table(p, L, [100] * 4, 1199)
    bad = L.copy()
    bad[1, 2] = np.nan
    with pytest.raises(mpe.MpeError):
        mpe.allocate_bits_table(p, bad, [100] * 4, 2000)
    with pytest.raises(ValueError):
        mpe.allocate_bits_table(p, L[:3], [100] * 4, 2000)


def test_repage_with_measured_allocator():
    wl = synth.scaled(synth.WORKLOADS[1], E=8, H=256, F=256)
    p = synth.importance(wl)
    W = [wl.W_e] * wl.E
    masters = [synth.expert_weights(wl, e, device="cuda") for e in range(wl.E)]
    # experts of different sensitivity: scale some masters up
    for e in (1, 4):
        masters[e] = (masters[e].float() * 8).half()
    cpu = [m.cpu().numpy() for m in masters]
    loss = np.array([[oq.quantization_mse(cpu[e], b) for b in WIDTHS] for e in range(wl.E)])
    pool = wl.E * op.pages_needed(8, wl.H, wl.F)
    ctx = mpe.Context(wl.E, wl.H, wl.F, pool_pages=pool)
    ctx.set_allocator(mpe.ALLOCATOR_MEASURED)
    alloc = op.PageAllocator(pool, wl.E, wl.H, wl.F)
    bits0 = np.full(wl.E, 8, np.uint8)
    ctx.quantize_experts(masters, bits0)
    alloc.place(bits0)
    for avg in [6.0, 4.0, 3.0, 5.0, 3.5]:
        B = synth.budget_for(wl, avg)
        n = ctx.repage(B, p)
        nb = oa.allocate_bits_table(p, loss, W, B)
        assert n == len(alloc.repage(nb))
        assert np.array_equal(ctx.bits(), nb)
        for e in range(wl.E):
            assert np.array_equal(ctx.expert_stream(e),
                                  OracleExpert(cpu[e], wl.H, wl.F, int(nb[e])).stream())
    assert np.array_equal(ctx.measure_loss(), loss)
