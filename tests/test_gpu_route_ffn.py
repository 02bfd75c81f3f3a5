"""GPU parity for token bucketing (bit-exact) and for the routed SwiGLU expert
FFN run from the pages (rel-Frobenius <= 5e-3, max-abs <= 2e-2 * max|oracle|)
against the float64 dequantize-then-multiply oracle (PagedWeight, "Dynamic
Paging")."""
import numpy as np
import pytest
import torch

import synth
from oracle import route as orr

from _helpers import OracleExpert, check_ffn, oracle_moe

pytestmark = pytest.mark.gpu

mpe = pytest.importorskip("mixed_precision_expert_b200")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixed_precision_expert_b200.build import build
    build()
    assert torch.cuda.is_available()


@pytest.mark.parametrize("T,k,E,seed", [(1, 1, 8, 0), (64, 2, 8, 1), (64, 8, 128, 2),
                                        (128, 8, 256, 3), (100, 7, 33, 4), (1000, 8, 128, 5),
                                        (8192, 8, 128, 6), (3000, 3, 1024, 7)])
def test_route_parity(T, k, E, seed):
    rng = np.random.default_rng(seed)
    ids = rng.integers(0, E, size=(T, k)).astype(np.int32)
    if seed % 2:
        ids[rng.integers(0, T, 3), rng.integers(0, k, 3)] = rng.choice([-5, E, E + 7], 3)
    ctx = mpe.Context(E, 128, 128)
    perm, offs, inv = ctx.route(torch.from_numpy(ids).cuda())
    rp, ro, ri = orr.route(ids, E)
    assert np.array_equal(offs.cpu().numpy(), ro)
    n = int(ro[-1])
    assert np.array_equal(perm.cpu().numpy()[:n], rp)
    assert np.array_equal(inv.cpu().numpy(), ri)
    bad = bool((ids < 0).any() or (ids >= E).any())
    assert bool(ctx.status(clear=True) & mpe.STATUS_BAD_EXPERT_ID) == bad


def test_route_and_forward_reject_too_many_assignments():
    # T*k above MPE_MAX_ASSIGNMENTS (2^24) is refused before any device work
    # (the work-group counts of the bucketing live in 21-bit scan fields)
    L = mpe.lib()
    ctx = mpe.Context(8, 128, 128)
    buf = torch.zeros(16, dtype=torch.int32, device="cuda")
    rc = L.mpe_route(ctx._h, buf.data_ptr(), (1 << 20) + 1, 16, buf.data_ptr(), buf.data_ptr(),
                     buf.data_ptr())
    assert rc == -1 and b"exceeds" in L.mpe_last_error(ctx._h)
    rc = L.mpe_moe_ffn(ctx._h, buf.data_ptr(), (1 << 20) + 1, buf.data_ptr(), buf.data_ptr(), 16,
                       buf.data_ptr())
    assert rc == -1
    ctx.close()


def _layer(wl, bits=None, device="cuda", path=0):
    if bits is None:
        bits = mpe.allocate_bits(synth.importance(wl), [wl.W_e] * wl.E, wl.budget_bits)
    masters = [synth.expert_weights(wl, e, device=device) for e in range(wl.E)]
    ctx = mpe.Context(wl.E, wl.H, wl.F, path=path)
    ctx.quantize_experts(masters, bits)
    ox = [OracleExpert(m.cpu().numpy(), wl.H, wl.F, int(b)) for m, b in zip(masters, bits)]
    mats = {}

    def mats_of(e):
        if e not in mats:
            mats[e] = ox[e].mats()
        return mats[e]

    return ctx, masters, mats_of


def _run(ctx, x, ids, w):
    out = ctx.moe_ffn(x.cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    # no bounded device wait may have run out (that would mean a lost stage)
    assert not (ctx.status() & mpe.STATUS_WAIT_TIMEOUT)
    return out.double().cpu().numpy()


def test_ffn_tiny_layer():
    wl = synth.WORKLOADS[1]
    ctx, _, mats_of = _layer(wl)
    ids, w = synth.routing(wl)
    x = synth.activations(wl)
    got = _run(ctx, x, ids, w)
    check_ffn(got, oracle_moe(x, ids, w, mats_of, wl.E))
    assert ctx.status() == 0


@pytest.mark.parametrize("bits", [(3,) * 4, (4,) * 4, (8,) * 4, (3, 4, 8, 3)])
def test_ffn_each_width(bits):
    wl = synth.scaled(synth.WORKLOADS[1], E=4, H=384, F=256, T=19, k=2)
    ctx, _, mats_of = _layer(wl, np.array(bits, np.uint8))
    ids, w = synth.routing(wl)
    x = synth.activations(wl)
    check_ffn(_run(ctx, x, ids, w), oracle_moe(x, ids, w, mats_of, wl.E))


def test_ffn_edge_token_counts():
    wl = synth.scaled(synth.WORKLOADS[1], E=6, H=256, F=384, T=40, k=3)
    ctx, _, mats_of = _layer(wl, np.array([3, 4, 8, 4, 3, 8], np.uint8))
    x = synth.activations(wl)
    rng = np.random.default_rng(3)
    cases = []
    # a single token
    cases.append((x[:1], np.array([[2, 0, 5]], np.int32)))
    # every token on expert 1 (more than one 16-token work group), expert 4 unused
    ids = np.stack([np.ones(40, np.int32), rng.integers(0, 4, 40).astype(np.int32),
                    np.full(40, 5, np.int32)], 1)
    cases.append((x, ids))
    # 17 tokens: a ragged last n-tile and work group
    ids = rng.integers(0, 6, size=(17, 3)).astype(np.int32)
    cases.append((x[:17], ids))
    for xi, ids in cases:
        w = rng.random(ids.shape).astype(np.float32)
        check_ffn(_run(ctx, xi.contiguous(), ids, w), oracle_moe(xi, ids, w, mats_of, wl.E))


def test_ffn_invalid_ids_are_dropped():
    wl = synth.scaled(synth.WORKLOADS[1], E=4, H=128, F=256, T=5, k=2)
    ctx, _, mats_of = _layer(wl, np.array([4, 4, 8, 3], np.uint8))
    x = synth.activations(wl)
    ids = np.array([[0, 9], [1, -1], [2, 3], [4, 0], [3, 3]], np.int32)
    w = np.full(ids.shape, 0.5, np.float32)
    got = _run(ctx, x, ids, w)
    assert ctx.status(clear=True) & mpe.STATUS_BAD_EXPERT_ID
    check_ffn(got, oracle_moe(x, ids, w, mats_of, wl.E))


def test_ffn_zero_tokens_is_a_no_op():
    wl = synth.scaled(synth.WORKLOADS[1], E=2, H=128, F=128)
    ctx, _, _ = _layer(wl, np.array([4, 4], np.uint8))
    out = ctx.moe_ffn(torch.empty(0, 128, dtype=torch.bfloat16, device="cuda"),
                      torch.empty(0, 2, dtype=torch.int32, device="cuda"),
                      torch.empty(0, 2, dtype=torch.float32, device="cuda"))
    assert out.shape == (0, 128)


def test_ffn_host_buffers_match_device_call():
    wl = synth.WORKLOADS[1]
    ctx, _, _ = _layer(wl)
    ids, w = synth.routing(wl)
    x = synth.activations(wl)
    dev = _run(ctx, x, ids, w)
    xh = x.pin_memory()
    idh = torch.from_numpy(ids).pin_memory()
    wh = torch.from_numpy(w).pin_memory()
    oh = torch.empty(x.shape, dtype=torch.bfloat16).pin_memory()
    ctx.moe_ffn_host(xh, idh, wh, oh)
    assert np.array_equal(oh.double().numpy(), dev)


def _host_call(ctx, x, ids, w):
    xh = x.pin_memory()
    idh = torch.from_numpy(ids).pin_memory()
    wh = torch.from_numpy(w).pin_memory()
    oh = torch.empty(x.shape, dtype=torch.bfloat16).pin_memory()
    ctx.moe_ffn_host(xh, idh, wh, oh)
    return oh.double().numpy()


@pytest.mark.parametrize("path", [1, 2])
def test_ffn_host_graph_replay_matches_device_call(path):
    # the host-buffer call sizes its buffers on the first call with a shape,
    # captures its kernels as a CUDA graph on the second and replays it on
    # later ones: every call must equal the device-pointer call bit for bit,
    # also across a repage (new widths, same buffers) and a compensation switch
    wl = synth.scaled(synth.WORKLOADS[3], E=16, T=48, k=4)
    ctx, masters, _ = _layer(wl, path=path)
    p = synth.importance(wl)
    for step in range(7):
        if step == 3:
            ctx.repage(synth.budget_for(wl, 3.2), p)
        if step == 5 and path == 1:
            ctx.set_compensation(8)
        ids, w = synth.routing(wl, seed=50 + step)
        x = synth.activations(wl, seed=50 + step)
        got = _host_call(ctx, x, ids, w)
        assert np.array_equal(got, _run(ctx, x, ids, w)), step
    assert ctx.status() == 0


def test_split_k_forward_is_deterministic_across_forwards():
    # gate/up of this shape runs in two K parts (8 block columns, 3 tile
    # groups per work group) whose partials are summed in part order:
    # repeated forwards must give the same bits, other batches in between
    # included, and match the oracle
    wl = synth.scaled(synth.WORKLOADS[1], E=8, H=1024, F=512, T=16, k=2)
    ctx, _, mats_of = _layer(wl)
    ids, w = synth.routing(wl, seed=3)
    x = synth.activations(wl, seed=3)
    first = _run(ctx, x, ids, w)
    check_ffn(first, oracle_moe(x, ids, w, mats_of, wl.E))
    for _ in range(3):
        assert np.array_equal(_run(ctx, x, ids, w), first)
    ids2, w2 = synth.routing(wl, seed=4)
    x2 = synth.activations(wl, seed=4)
    check_ffn(_run(ctx, x2, ids2, w2), oracle_moe(x2, ids2, w2, mats_of, wl.E))
    assert np.array_equal(_run(ctx, x, ids, w), first)
    assert ctx.status() == 0


@pytest.mark.parametrize("path", [1, 2])
def test_ffn_host_async_pipeline_matches_device_call(path):
    # queued host-buffer calls (two staging slots taken in turn, copies on
    # their own stream) give, call by call, the device-pointer call's bits:
    # five calls in flight before the first wait, a shape change, and a
    # repage queued on the context stream between two queued calls
    wl = synth.scaled(synth.WORKLOADS[3], E=16, T=48, k=4)
    ctx, _, _ = _layer(wl, path=path)
    p = synth.importance(wl)
    calls = []
    for step in range(9):
        T = wl.T if step != 6 else 20
        w2 = synth.scaled(wl, T=T)
        ids, w = synth.routing(w2, seed=80 + step)
        x = synth.activations(w2, seed=80 + step)
        calls.append((x, ids, w))
    hostbuf = []
    for x, ids, w in calls:
        hostbuf.append((x.pin_memory(), torch.from_numpy(ids).pin_memory(),
                        torch.from_numpy(w).pin_memory(),
                        torch.empty(x.shape, dtype=torch.bfloat16).pin_memory()))
    tickets = []
    for i in range(5):
        xh, ih, wh, oh = hostbuf[i]
        tickets.append(ctx.moe_ffn_host_async(xh, ih, wh, oh))
    assert tickets == sorted(tickets) and len(set(tickets)) == 5
    for t in tickets:
        ctx.wait_host(t)
    want = [_run(ctx, *c) for c in calls[:5]]
    for i in range(5):
        assert np.array_equal(hostbuf[i][3].double().numpy(), want[i]), i
    # a repage between queued calls: the call queued after it sees the new widths
    t5 = ctx.moe_ffn_host_async(*hostbuf[5])
    ctx.repage(synth.budget_for(wl, 3.2), p)
    t6 = ctx.moe_ffn_host_async(*hostbuf[6])
    t7 = ctx.moe_ffn_host_async(*hostbuf[7])
    t8 = ctx.moe_ffn_host_async(*hostbuf[8])
    for t in (t5, t6, t7, t8):
        ctx.wait_host(t)
    for i in (6, 7, 8):
        assert np.array_equal(hostbuf[i][3].double().numpy(), _run(ctx, *calls[i])), i
    assert ctx.status() == 0


def test_ffn_host_async_tickets():
    wl = synth.scaled(synth.WORKLOADS[1], E=4, H=256, F=256, T=8, k=2)
    ctx, _, _ = _layer(wl)
    ids, w = synth.routing(wl)
    x = synth.activations(wl)
    with pytest.raises(mpe.MpeError):
        ctx.wait_host(0)  # nothing issued yet
    buf = (x.pin_memory(), torch.from_numpy(ids).pin_memory(), torch.from_numpy(w).pin_memory(),
           torch.empty(x.shape, dtype=torch.bfloat16).pin_memory())
    t = ctx.moe_ffn_host_async(*buf)
    with pytest.raises(mpe.MpeError):
        ctx.wait_host(t + 1)
    ctx.wait_host(t)
    ctx.wait_host(t)  # waiting again is harmless
    empty = (buf[0][:0], buf[1][:0], buf[2][:0], buf[3][:0])
    assert ctx.moe_ffn_host_async(*empty) == 2**64 - 1
    ctx.wait_host(2**64 - 1)
    assert np.array_equal(buf[3].double().numpy(), _run(ctx, x, ids, w))


def test_ffn_finegrained_decode_full_size():
    # 128 experts, hidden 2048, ffn 768, 64 tokens top-8 (Zipf-skewed), 3.5 bits average
    wl = synth.WORKLOADS[3]
    ctx, _, mats_of = _layer(wl)
    ids, w = synth.routing(wl)
    x = synth.activations(wl)
    got = _run(ctx, x, ids, w)
    toks = np.arange(0, wl.T, 4)
    check_ffn(got[toks], oracle_moe(x, ids, w, mats_of, wl.E, tokens=toks))


def test_bounded_wait_gives_up_and_context_stays_usable():
    # a device wait that nothing completes gives up after its limit and
    # reports STATUS_WAIT_TIMEOUT; the context then serves a forward pass
    wl = synth.scaled(synth.WORKLOADS[1], E=4, H=256, F=256, T=8, k=2)
    ctx, _, mats_of = _layer(wl, np.array([3, 4, 8, 4], np.uint8))
    assert ctx.status() == 0
    ctx.selftest_wait(5_000_000)  # 5 ms
    assert ctx.status(clear=True) & mpe.STATUS_WAIT_TIMEOUT
    assert ctx.status() == 0
    ids, w = synth.routing(wl)
    x = synth.activations(wl)
    check_ffn(_run(ctx, x, ids, w), oracle_moe(x, ids, w, mats_of, wl.E))
    with pytest.raises(mpe.MpeError):
        ctx.selftest_wait(0)
