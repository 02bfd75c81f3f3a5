"""Pins for oracle.prefix, the prefix-compatible (nested-grid) quantizer and
its layered page store.

The grid is checked by exact rational arithmetic over every finite fp16
weight for several absmax values (each code's bin holds its weight), by a
hand-worked example and by its bounds; the layers by the location of every
bit of sampled codes, recomputed with scalar index arithmetic, a hand-worked
word and round trips; the page rules by their
invariants (disjoint pages, dropped layers freed without encoding, unchanged
layers kept, all-or-nothing on shortage).
"""
from fractions import Fraction

import numpy as np
import pytest

from oracle import prefix as X


def test_hand_worked_codes():
    w = np.array([0.5, -1.0, 1.0, 0.0, -2.0 ** -24, 0.25], dtype=np.float16)
    m, u8 = X.prefix_codes(w)
    assert m == 1.0
    # 128 w / m = 64, -128, 128 (clamped), 0, just below 0, 32
    assert list(u8) == [192, 0, 255, 128, 127, 160]
    assert list(X.code_of_width(u8, 3)) == [6, 0, 7, 4, 3, 5]
    assert list(X.dequantize(m, X.code_of_width(u8, 3), 3)) == [0.625, -0.875, 0.875, 0.125,
                                                                -0.125, 0.375]
    assert X.dequantize(m, np.array([0, 255]), 8).tolist() == [-255 / 256, 255 / 256]


def _all_fp16_upto(m):
    bits = np.arange(0, 0x7C00, dtype=np.uint16)
    v = bits.view(np.float16)
    v = v[v.astype(np.float64) <= m]
    return np.concatenate([v, -v]).astype(np.float16)


@pytest.mark.parametrize("m", [1.0, 0.2001953125, 3.0, 65504.0, 6.103515625e-05])
def test_every_fp16_weight_lies_in_its_bins(m):
    w = _all_fp16_upto(m)
    w = np.concatenate([w, np.array([m], np.float16)])
    mm, u8 = X.prefix_codes(w)
    assert mm == float(np.float16(m))
    M = Fraction(mm)
    rng = np.random.default_rng(0)
    sample = rng.choice(len(w), size=min(len(w), 3000), replace=False)
    for i in sample:
        q = Fraction(float(w[i])) * 128 / M
        want = max(0, min(255, (q.numerator // q.denominator) + 128))
        assert u8[i] == want
    for b in (3, 4, 8):
        ub = X.code_of_width(u8, b)
        lo = -mm + ub * (2 * mm / 2 ** b)
        hi = lo + 2 * mm / 2 ** b
        wd = w.astype(np.float64)
        assert np.all(lo <= wd) and np.all((wd < hi) | (wd == mm))
        err = np.abs(wd - X.dequantize(mm, ub, b))
        assert np.all(err <= mm / 2 ** b)
    order = np.argsort(w.astype(np.float64), kind="stable")
    assert np.all(np.diff(u8[order]) >= 0)  # codes never decrease as w grows


def test_zero_master_and_nonfinite():
    m, u8 = X.prefix_codes(np.zeros(64, np.float16))
    assert m == 0.0 and np.all(u8 == 128)
    assert np.all(X.dequantize(m, X.code_of_width(u8, 3), 3) == 0.0)
    with pytest.raises(ValueError):
        X.prefix_codes(np.array([1.0, np.inf], np.float16))


def test_layers_compose_the_codes():
    u8 = np.arange(256)
    A, B, C = (X.layer_values(u8, L) for L in "ABC")
    assert np.array_equal(32 * A + 16 * B + C, u8)
    assert np.array_equal(A, X.code_of_width(u8, 3))
    assert np.array_equal(2 * A + B, X.code_of_width(u8, 4))


def _code_bits(layer, mat, r, k, H, F):
    """(byte offset of the word, bit in the word, bit of the code) for every
    bit of code (r, k) of matrix mat (0 = W1, 1 = W3, 2 = W2) in a layer's
    chunk stream, by scalar index arithmetic: chunks of 16 rows x 128 codes,
    W1 / W3 chunks alternating, then W2 with tile pairs alternating by block
    column; a row's 128 codes as four quarters of 32."""
    b = X.LAYER_BITS[layer]
    K = H if mat < 2 else F
    tau, rho = divmod(r, 16)
    j, i = divmod(k, 128)
    q, ip = divmod(i, 32)
    nc1 = (F // 16) * (H // 128)
    if mat < 2:
        chunk = 2 * (tau * (K // 128) + j) + mat
    else:
        chunk = 2 * nc1 + 2 * ((tau // 2) * (K // 128) + j) + (tau % 2)
    base = chunk * 256 * b + rho * 16 * b + q * 4 * b
    if b == 3 and ip >= 30:
        top = 15 if ip == 30 else 31
        return [(base + 4 * n, top, n) for n in range(3)]
    per = 10 if b == 3 else 32 // b
    w, ii = divmod(ip, per)
    pos = 16 * (ii & 1) + b * (ii >> 1)
    return [(base + 4 * w, pos + n, n) for n in range(b)]


@pytest.mark.parametrize("layer", ["A", "B", "C"])
def test_layer_stream_element_locations(layer):
    H, F = 256, 256  # W2 with two block columns
    rng = np.random.default_rng(1)
    u8 = rng.integers(0, 256, size=3 * H * F)
    s = X.layer_stream(u8, layer, H, F)
    b = X.LAYER_BITS[layer]
    assert s.shape == (3 * (F // 16) * (H // 128), 256 * b)
    assert s.size * 8 == 3 * H * F * b
    flat = s.reshape(-1)
    vals = X.layer_values(u8, layer)
    mats = [(0, F, H, 0), (1, F, H, F * H), (2, H, F, 2 * F * H)]
    for mat, R, K, off in mats:
        rows = rng.choice(R, size=12, replace=False)
        for r in rows:
            for k in range(K):
                got = 0
                for byte, bit, n in _code_bits(layer, mat, int(r), k, H, F):
                    word = int.from_bytes(flat[byte:byte + 4].tobytes(), "little")
                    got |= ((word >> bit) & 1) << n
                assert got == vals[off + r * K + k], (layer, mat, r, k)
    assert np.array_equal(X.layer_codes(s, layer, H, F), vals)


def test_layer_b_hand_word():
    # the one-bit quarter: c'_i at bit 16 (i & 1) + (i >> 1). Codes 1 at
    # i = 0, 1, 30, 31 give bits 0, 16, 15, 31 -> 0x80018001.
    H, F = 128, 128
    u8 = np.zeros(3 * H * F, dtype=np.int64)
    for i in (0, 1, 30, 31):
        u8[i] = 16  # B = bit 4 of u8
    s = X.layer_stream(u8, "B", H, F)
    assert int.from_bytes(s.reshape(-1)[:4].tobytes(), "little") == 0x80018001
    assert int(s.reshape(-1)[4:].astype(np.int64).sum()) == 0


def test_page_rules():
    H, F, P = 256, 128, 4096
    W_e = 3 * H * F
    n = {L: X.layer_pages(L, H, F, P) for L in "ABC"}
    assert n == {"A": 10, "B": 3, "C": 12}  # 48 chunks at 5 / 16 / 4 per page
    pool = 4 * (n["A"] + n["B"] + n["C"])
    lp = X.LayeredPages(pool, 4, H, F, P)
    enc = lp.place([8, 3, 4, 8])
    assert enc == {0: ["A", "B", "C"], 1: ["A"], 2: ["A", "B"], 3: ["A", "B", "C"]}
    before = {e: dict(lp.pages[e]) for e in range(4)}
    enc = lp.repage([3, 3, 8, 4])
    # 0: 8 -> 3 drops B, C (nothing encoded); 2: 4 -> 8 adds C; 3: 8 -> 4 drops C
    assert enc == {2: ["C"]}
    assert lp.pages[0] == {"A": before[0]["A"]}
    assert lp.pages[1] == before[1]
    assert lp.pages[2]["A"] == before[2]["A"] and lp.pages[2]["B"] == before[2]["B"]
    used = [p for e in range(4) for L in lp.pages[e] for p in lp.pages[e][L]]
    assert len(used) == len(set(used)) == int((~lp.free).sum())
    # C of expert 2 takes the lowest pages freed by 0 and 3 (releases come first)
    freed = sorted(before[0]["B"] + before[0]["C"] + before[3]["C"])
    assert lp.pages[2]["C"] == freed[:n["C"]]
    assert X.repage_bytes(enc, W_e) == 2 * W_e + W_e // 2
    first, npg, idx = lp.table()
    assert npg.tolist() == [10, 10, 25, 13]
    # shortage: nothing changes
    snap = ([dict(p) for p in lp.pages], lp.free.copy(), lp.bits.copy())
    lp2 = X.LayeredPages(n["A"] * 4 + n["B"], 4, H, F, P)
    lp2.place([3, 3, 3, 3])
    with pytest.raises(X.PoolExhausted):
        lp2.repage([8, 3, 3, 3])
    assert lp2.bits.tolist() == [3, 3, 3, 3] and int((~lp2.free).sum()) == 4 * n["A"]
