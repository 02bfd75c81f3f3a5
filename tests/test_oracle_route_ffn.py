"""Pins for oracle.route (token-to-expert bucketing) and oracle.ffn (the
dequantize-then-multiply SwiGLU expert FFN with top-k combine).

Route: brute-force bucketing by plain loops on small inputs. FFN: pure-Python
triple loops on tiny shapes, and special cases -- all-zero codes give zero
output, a one-hot token reads one column of the gate matrix, 8-bit codes of
weights that are exact multiples of the scale dequantize losslessly, and the
combine is linear in the top-k weights.
"""
import math

import numpy as np
import pytest

from oracle import ffn as Fn
from oracle import quantize as Qz
from oracle import route as Rt


def brute_route(ids, E):
    flat = [int(x) for x in np.asarray(ids).ravel()]
    buckets = [[] for _ in range(E)]
    for a, e in enumerate(flat):
        if 0 <= e < E:
            buckets[e].append(a)
    perm = [a for b in buckets for a in b]
    offs = [0]
    for b in buckets:
        offs.append(offs[-1] + len(b))
    inv = [-1] * len(flat)
    for pos, a in enumerate(perm):
        inv[a] = pos
    return perm, offs, inv


@pytest.mark.parametrize("seed", range(8))
def test_route_brute_force(seed):
    rng = np.random.default_rng(seed)
    E = int(rng.integers(1, 20))
    T, k = int(rng.integers(0, 40)), int(rng.integers(1, 9))
    ids = rng.integers(-1, E + 1, size=(T, k)).astype(np.int32)  # includes invalid ids
    perm, offs, inv = Rt.route(ids, E)
    bp, bo, bi = brute_route(ids, E)
    assert list(perm) == bp and list(offs) == bo and list(inv) == bi


def test_route_properties_all_one_expert():
    ids = np.full((64, 8), 5, np.int32)
    perm, offs, inv = Rt.route(ids, 128)
    assert list(perm) == list(range(512))            # stable: identity
    assert offs[5] == 0 and offs[6] == 512 and offs[-1] == 512
    assert np.array_equal(inv, np.arange(512))


def loop_expert_ffn(x, w1, w3, w2):
    n, H = len(x), len(x[0])
    F = len(w1)
    out = []
    for t in range(n):
        h = []
        for f in range(F):
            g = 0.0
            v = 0.0
            for c in range(H):
                g += w1[f][c] * x[t][c]
                v += w3[f][c] * x[t][c]
            h.append(g / (1.0 + math.exp(-g)) * v)
        y = []
        for r in range(H):
            acc = 0.0
            for f in range(F):
                acc += w2[r][f] * h[f]
            y.append(acc)
        out.append(y)
    return np.array(out)


def test_expert_ffn_triple_loop():
    rng = np.random.default_rng(0)
    n, H, F = 3, 6, 5
    x = rng.standard_normal((n, H))
    w1, w3 = rng.standard_normal((F, H)), rng.standard_normal((F, H))
    w2 = rng.standard_normal((H, F))
    np.testing.assert_allclose(Fn.expert_ffn(x, w1, w3, w2),
                               loop_expert_ffn(x.tolist(), w1.tolist(), w3.tolist(), w2.tolist()),
                               rtol=1e-12, atol=1e-12)


def test_moe_ffn_loop_combine():
    rng = np.random.default_rng(1)
    T, H, F, E, k = 5, 4, 3, 3, 2
    x = rng.standard_normal((T, H))
    mats = [(rng.standard_normal((F, H)), rng.standard_normal((F, H)), rng.standard_normal((H, F)))
            for _ in range(E)]
    ids = np.array([[0, 1], [2, 0], [1, 1], [2, 2], [0, 2]], np.int32)
    w = rng.random((T, k)).astype(np.float32)
    out = Fn.moe_ffn(x, ids, w, lambda e: mats[e], E)
    for t in range(T):
        ref = np.zeros(H)
        for j in range(k):
            e = ids[t, j]
            ref += float(w[t, j]) * loop_expert_ffn([x[t].tolist()], *(m.tolist() for m in mats[e]))[0]
        np.testing.assert_allclose(out[t], ref, rtol=1e-12, atol=1e-12)
    sub = Fn.moe_ffn(x, ids, w, lambda e: mats[e], E, tokens=[3, 1])
    np.testing.assert_allclose(sub, out[[3, 1]], rtol=1e-13, atol=1e-13)


def test_all_zero_codes_give_zero_output():
    H, F = 8, 4
    z = Qz.dequantize(np.zeros((F, H), np.int64), np.float32(0.01))
    z2 = Qz.dequantize(np.zeros((H, F), np.int64), np.float32(0.01))
    x = np.random.default_rng(2).standard_normal((3, H))
    assert np.all(Fn.expert_ffn(x, z, z, z2) == 0.0)


def test_one_hot_token_reads_gate_column():
    rng = np.random.default_rng(3)
    H, F, b = 16, 8, 4
    k1 = rng.integers(-7, 8, size=(F, H))
    s = np.float32(0.0123)
    w1 = Qz.dequantize(k1, s)
    x = np.zeros((1, H))
    x[0, 5] = 1.0
    g, v = Fn.gate_up(x, w1, w1)
    np.testing.assert_array_equal(g[0], float(s) * k1[:, 5])


def test_8bit_exact_multiples_dequantize_losslessly():
    # fp16 weights that are integer multiples of s = 2^-7 with |k| <= 127 and max
    # |w| = 127 s: 8-bit quantization returns exactly the fp16 master, so the
    # quantized FFN equals the FFN of the master weights
    rng = np.random.default_rng(4)
    H, F = 16, 8
    k = rng.integers(-127, 128, size=3 * H * F)
    k[0] = 127
    w = (k * 2.0 ** -7).astype(np.float16)
    m, s, kk = Qz.quantize_expert(w, 8)
    assert float(s) == 2.0 ** -7 and np.array_equal(kk, k)
    deq = Qz.dequantize(kk, s)
    assert np.array_equal(deq, w.astype(np.float64))
    x = rng.standard_normal((2, H))
    w64 = w.astype(np.float64)
    a = Fn.expert_ffn(x, deq[:F * H].reshape(F, H), deq[F * H:2 * F * H].reshape(F, H),
                      deq[2 * F * H:].reshape(H, F))
    bb = Fn.expert_ffn(x, w64[:F * H].reshape(F, H), w64[F * H:2 * F * H].reshape(F, H),
                       w64[2 * F * H:].reshape(H, F))
    np.testing.assert_array_equal(a, bb)


def test_combine_is_linear_in_topk_weights():
    rng = np.random.default_rng(5)
    T, H, F, E, k = 6, 8, 4, 4, 2
    x = rng.standard_normal((T, H))
    mats = [(rng.standard_normal((F, H)), rng.standard_normal((F, H)), rng.standard_normal((H, F)))
            for _ in range(E)]
    ids = rng.integers(0, E, size=(T, k))
    wa = rng.random((T, k))
    wb = rng.random((T, k))
    f = lambda w: Fn.moe_ffn(x, ids, w, lambda e: mats[e], E)
    np.testing.assert_allclose(f(wa + wb), f(wa) + f(wb), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(f(2.0 * wa), 2.0 * f(wa), rtol=1e-12, atol=1e-12)


def test_invalid_ids_contribute_nothing():
    rng = np.random.default_rng(6)
    T, H, F, E = 2, 4, 2, 2
    x = rng.standard_normal((T, H))
    mats = [(rng.standard_normal((F, H)), rng.standard_normal((F, H)), rng.standard_normal((H, F)))
            for _ in range(E)]
    w = np.ones((T, 2))
    a = Fn.moe_ffn(x, np.array([[0, 7], [1, -1]]), w, lambda e: mats[e], E)
    b = Fn.moe_ffn(x, np.array([[0, 0], [1, 1]]), np.array([[1.0, 0.0], [1.0, 0.0]]),
                   lambda e: mats[e], E)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)
