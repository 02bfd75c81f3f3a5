"""Pins for oracle.compensate (DecDEC summary, 3.1-3.2 and Figure 4).

The channel choice is checked against a plain sort, the compensated linear
against a hand-worked example and against an explicit mask matrix, and the
layer against its two closed-form ends: no channel is the plain quantized
layer, every channel is the fp16-weight layer. Figure 4's observation (sorted
by |x| beats random order) is checked on a synthetic expert whose activations
carry outlier channels.
"""
import numpy as np
import pytest

from oracle import compensate as C
from oracle import ffn as of
from oracle import quantize as oq


def test_salient_channels_brute_force():
    rng = np.random.default_rng(0)
    for _ in range(200):
        L = int(rng.integers(1, 40))
        row = rng.integers(-4, 5, size=L).astype(np.float64) * 0.5  # many ties
        n = int(rng.integers(0, L + 3))
        ranked = sorted(range(L), key=lambda c: (-abs(row[c]), c))
        want = sorted(ranked[:n]) if n < L else list(range(L))
        assert list(C.salient_channels(row, n)) == want


def test_hand_worked_linear():
    w = np.array([[0.5, 0.25, -1.0], [1.0, 0.0, 0.75]])
    w_hat = np.array([[0.5, 0.0, -1.0], [1.0, 0.5, 1.0]])
    x = np.array([1.0, -4.0, 2.0])
    # |x| = 1, 4, 2: one channel -> {1}; two -> {1, 2}
    assert list(C.compensated_linear(w_hat, w, x, 0)) == [-1.5, 1.0]
    assert list(C.compensated_linear(w_hat, w, x, 1)) == [-2.5, 3.0]
    assert list(C.compensated_linear(w_hat, w, x, 2)) == [-2.5, 2.5]
    assert list(w @ x) == [-2.5, 2.5]


def test_linear_equals_mask_matrix():
    rng = np.random.default_rng(1)
    w = rng.standard_normal((24, 40))
    w_hat = np.round(w * 4) / 4
    for n in (0, 1, 5, 17, 40):
        x = rng.standard_normal(40)
        M = np.zeros_like(w)
        M[:, C.salient_channels(x, n)] = 1.0
        want = (w_hat + (w - w_hat) * M) @ x
        np.testing.assert_allclose(C.compensated_linear(w_hat, w, x, n), want, rtol=1e-12,
                                   atol=1e-12)


def _tiny_layer(seed=3, E=3, H=48, F=32, b=3):
    rng = np.random.default_rng(seed)
    masters, hats = {}, {}
    for e in range(E):
        m = (rng.standard_normal(3 * H * F) * 0.02).astype(np.float16)
        _, s, k = oq.quantize_expert(m, b)
        d = oq.dequantize(k, s)
        f = m.astype(np.float64)
        split = lambda a: (a[:F * H].reshape(F, H), a[F * H:2 * F * H].reshape(F, H),
                           a[2 * F * H:].reshape(H, F))
        masters[e], hats[e] = split(f), split(d)
    T, k = 6, 2
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)])
    w = rng.dirichlet(np.ones(k), size=T)
    x = rng.standard_normal((T, H))
    x[:, [3, 17]] *= 20.0  # outlier channels
    return masters, hats, x, ids, w, E, H, F


def test_layer_ends():
    masters, hats, x, ids, w, E, H, F = _tiny_layer()
    plain = of.moe_ffn(x, ids, w, lambda e: hats[e], E)
    got0 = C.moe_ffn_compensated(x, ids, w, lambda e: hats[e], lambda e: masters[e], E, 0)
    np.testing.assert_allclose(got0, plain, rtol=1e-12, atol=1e-15)
    full = of.moe_ffn(x, ids, w, lambda e: masters[e], E)
    got_all = C.moe_ffn_compensated(x, ids, w, lambda e: hats[e], lambda e: masters[e], E,
                                    max(H, F))
    np.testing.assert_allclose(got_all, full, rtol=1e-11, atol=1e-15)
    # in between: closer to the fp16-weight layer than the plain quantized one
    mid = C.moe_ffn_compensated(x, ids, w, lambda e: hats[e], lambda e: masters[e], E, 4)
    assert np.linalg.norm(mid - full) < np.linalg.norm(plain - full)


def test_figure4_sorted_beats_random():
    rng = np.random.default_rng(4)
    F, H = 256, 512
    m = (rng.standard_normal(F * H) * 0.02).astype(np.float16)
    _, s, k = oq.quantize_expert(m, 3)
    w = m.astype(np.float64).reshape(F, H)
    w_hat = oq.dequantize(k, s).reshape(F, H)
    x = rng.standard_normal(H)
    x[rng.choice(H, 8, replace=False)] *= 25.0
    by_mag = np.lexsort((np.arange(H), -np.abs(x)))
    rand = rng.permutation(H)
    es = C.error_curve(w_hat, w, x, by_mag)
    er = C.error_curve(w_hat, w, x, rand)
    assert es[0] == er[0] > 0.0
    for frac in (0.01, 0.02, 0.05):
        i = int(frac * H)
        assert es[i] < 0.5 * er[i], (frac, es[i], er[i])
    assert es[-1] < 1e-25 and er[-1] < 1e-25
    # the curve at i channels is the compensated linear with i salient channels
    for i in (1, 5, 20):
        got = np.mean((C.compensated_linear(w_hat, w, x, i) - w @ x) ** 2)
        assert got == pytest.approx(es[i], rel=1e-9)


def test_valid_choice_check():
    row = np.array([0.1, -3.0, 2.0, 2.001, 0.5])
    assert C.is_valid_choice(row, C.salient_channels(row, 2), 2, 0.0)  # {1, 3}
    assert not C.is_valid_choice(row, [1, 2], 2, 0.0)      # 2.001 left out
    assert C.is_valid_choice(row, [1, 2], 2, 0.01)         # within the tolerance
    assert not C.is_valid_choice(row, [1, 1], 2, 1.0)      # not distinct
    assert C.is_valid_choice(row, [0, 1, 2, 3, 4], 9, 0.0)  # n >= len: everything
    # relative part: 2.001 - 2.0 = 1e-3 against rel * (2.001 + 2.0)
    assert C.is_valid_choice(row, [1, 2], 2, 0.0, rel=2.0 ** -8)     # 1e-3 <= 0.0156
    assert not C.is_valid_choice(row, [1, 2], 2, 0.0, rel=1e-4)      # 1e-3 > 4e-4
    assert C.is_valid_choice(row, [1, 2], 2, 6e-4, rel=1e-4)         # 1e-3 <= 6e-4 + 4e-4
    assert not C.is_valid_choice(row, [1, 4], 2, 0.0, rel=2.0 ** -8)  # 2.001 vs 0.5: far apart
    rng = np.random.default_rng(9)
    for _ in range(50):
        r = rng.standard_normal(30)
        n = int(rng.integers(1, 30))
        assert C.is_valid_choice(r, C.salient_channels(r, n), n, 0.0)


def test_down_masks_reproduce_own_choice():
    masters, hats, x, ids, w, E, H, F = _tiny_layer(seed=6)
    n = 5
    # the masks the oracle would choose itself, passed back in: same output
    masks = {}
    for t in range(ids.shape[0]):
        for j in range(ids.shape[1]):
            e = ids[t, j]
            w1h, w3h, _ = hats[e]
            w1, w3, _ = masters[e]
            g = C.compensated_linear(w1h, w1, x[t], n)
            v = C.compensated_linear(w3h, w3, x[t], n)
            masks[(t, j)] = C.salient_channels(of.silu(g) * v, n)
    a = C.moe_ffn_compensated(x, ids, w, lambda e: hats[e], lambda e: masters[e], E, n)
    b = C.moe_ffn_compensated(x, ids, w, lambda e: hats[e], lambda e: masters[e], E, n,
                              down_masks=masks)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-15)
