"""Pins for oracle.layout (the packed page format) and oracle.pages (page
allocator and page table; PagedWeight, "Dynamic Paging" and "Implementation
Details", memory management).

The words below were worked by hand from the layout definition in
oracle/layout.py; the element-location check recomputes every code's byte and
bit position with scalar index arithmetic, independently of the vectorised
packer.
"""
import numpy as np
import pytest

from oracle import layout as L
from oracle import pages as P


def block_words(u128, b):
    return L.pack_quarters(np.asarray(u128, dtype=np.uint32).reshape(4, 32), b).reshape(-1)


def test_hand_words_b4():
    # codes u_i = i mod 16. Quarter word 0 holds c'_0..c'_7 = 0..7 with c'_i at
    # bit 16(i&1) + 4(i>>1): low half nibbles 0,2,4,6 -> 0x6420, high half
    # 1,3,5,7 -> 0x7531. Word 1 holds 8..15 -> 0xECA8 | 0xFDB9 << 16.
    w = block_words(np.arange(128) % 16, 4)
    assert [int(x) for x in w[:4]] == [0x75316420, 0xFDB9ECA8, 0x75316420, 0xFDB9ECA8]
    assert np.all(w.reshape(4, 4) == w[:4])


def test_hand_words_b8():
    # codes u_i = i. Word w holds c'_{4w+i} at bit 16(i&1) + 8(i>>1): bytes
    # (c0, c2, c1, c3) -> 0x03010200; codes 4..7 -> 0x07050604; quarter 1
    # word 0 (codes 32..35) -> 0x23212220.
    w = block_words(np.arange(128), 8)
    assert int(w[0]) == 0x03010200 and int(w[1]) == 0x07050604
    assert int(w[8]) == 0x23212220
    assert int(w[31]) == 0x7F7D7E7C  # codes 124..127


def test_hand_words_b3():
    # codes u_i = i mod 8. Word v holds c'_{10v+i} at bit 16(i&1) + 3(i>>1), i < 10;
    # c'_30 = 6 = 0b110 and c'_31 = 7 = 0b111 give bit n of word n at bits 15 / 31.
    # word 0: low fields 0,2,4,6,0 -> 0x0D10; high 1,3,5,7,1 -> 0x1F59; spare
    #         bits (0 from c'_30, 1 from c'_31) -> 0x9F590D10
    # word 1: low 2,4,6,0,2 -> 0x21A2 (+0x8000); high 3,5,7,1,3 -> 0x33EB (+0x8000)
    # word 2: low 4,6,0,2,4 -> 0x4434 (+0x8000); high 5,7,1,3,5 -> 0x567D (+0x8000)
    w = block_words(np.arange(128) % 8, 3)
    assert [int(x) for x in w[:3]] == [0x9F590D10, 0xB3EBA1A2, 0xD67DC434]
    assert np.all(w.reshape(4, 3) == w[:3])


@pytest.mark.parametrize("b", [1, 3, 4, 8])
def test_quarter_roundtrip_and_size(b):
    rng = np.random.default_rng(b)
    u = rng.integers(0, 1 << b, size=(50, 32)).astype(np.uint32)
    words = L.pack_quarters(u, b)
    assert words.shape == (50, b)   # 32 codes * b bits = b words
    assert np.array_equal(L.unpack_quarters(words, b), u)
    with pytest.raises(ValueError):
        L.pack_quarters(np.full((1, 32), 1 << b), b)


def _location(r, k, K, b):
    """Byte offset of code (r, k) in a matrix chunk stream, and its bit positions.
    Returns (word byte offset, [(bit in word, bit of code)])."""
    tau, rho = divmod(r, 16)
    j, i = divmod(k, 128)
    q, ip = divmod(i, 32)
    chunk = tau * (K // 128) + j
    base = chunk * 256 * b + rho * 16 * b + q * 4 * b
    if b in (4, 8):
        per = 32 // b
        w, ii = divmod(ip, per)
        pos = 16 * (ii & 1) + b * (ii >> 1)
        return [(base + 4 * w, pos + n, n) for n in range(b)]
    if ip < 30:
        v, ii = divmod(ip, 10)
        pos = 16 * (ii & 1) + 3 * (ii >> 1)
        return [(base + 4 * v, pos + n, n) for n in range(3)]
    top = 15 if ip == 30 else 31
    return [(base + 4 * n, top, n) for n in range(3)]


@pytest.mark.parametrize("b", [3, 4, 8])
def test_matrix_element_locations(b):
    R, K = 32, 256
    rng = np.random.default_rng(10 + b)
    u = rng.integers(0, 1 << b, size=(R, K)).astype(np.uint32)
    s = L.pack_matrix(u, b)
    assert s.shape == (R // 16 * K // 128, 256 * b)
    assert s.size == R * K * b // 8
    flat = s.reshape(-1)
    for r in range(R):
        for k in range(K):
            val = 0
            for off, bit, n in _location(r, k, K, b):
                word = int.from_bytes(flat[off:off + 4].tobytes(), "little")
                val |= ((word >> bit) & 1) << n
            assert val == u[r, k]
    assert np.array_equal(L.unpack_matrix(s, R, K, b), u)


def test_expert_stream_order():
    H, F, b = 128, 32, 4
    u1 = np.full((F, H), 1, np.uint32)
    u3 = np.full((F, H), 2, np.uint32)
    u2 = np.full((H, F * 4), 3, np.uint32)[:, :F]  # [H, F] but F=32 is not a multiple of 128
    with pytest.raises(ValueError):
        L.expert_stream(u1, u3, u2, b)
    H, F = 128, 128
    u1 = np.full((F, H), 1, np.uint32)
    u3 = np.full((F, H), 2, np.uint32)
    u2 = np.full((H, F), 3, np.uint32)
    s = L.expert_stream(u1, u3, u2, b)
    n = L.n_chunks(H, F)
    assert s.shape[0] == n == 3 * (F // 16) * (H // 128)
    third = n // 3
    # constant codes -> every nibble equal; W1 and W3 chunks alternate, then W2
    assert np.all(s[0:2 * third:2] == 0x11) and np.all(s[1:2 * third:2] == 0x22)
    assert np.all(s[2 * third:] == 0x33)
    # distinct codes per matrix row: chunk 2c is W1's chunk c, 2c+1 is W3's
    # (F = 256: W2 has two block columns, so its column interleave shows)
    H, F = 256, 256
    rng = np.random.default_rng(1)
    u1 = rng.integers(0, 16, size=(F, H)).astype(np.uint32)
    u3 = rng.integers(0, 16, size=(F, H)).astype(np.uint32)
    u2 = rng.integers(0, 16, size=(H, F)).astype(np.uint32)
    s = L.expert_stream(u1, u3, u2, b)
    g1, g3 = L.pack_matrix(u1, b), L.pack_matrix(u3, b)
    for c in range(g1.shape[0]):
        assert np.array_equal(s[2 * c], g1[c]) and np.array_equal(s[2 * c + 1], g3[c])
    # W2: tiles 2v and 2v+1 alternate by block column
    g2 = L.pack_matrix(u2, b)
    nc1, nt2, nj2 = g1.shape[0], H // 16, F // 128
    for tau in range(nt2):
        for j in range(nj2):
            pos = 2 * nc1 + 2 * ((tau // 2) * nj2 + j) + (tau % 2)
            assert np.array_equal(s[pos], g2[tau * nj2 + j])
    # and the stream still carries every code exactly once
    assert sorted(map(bytes, s[2 * nc1:])) == sorted(map(bytes, g2))


# ----------------------------------------------------------------------------
# pages
# ----------------------------------------------------------------------------
def test_chunks_per_page():
    assert P.chunks_per_page(3) == 85 and P.chunks_per_page(4) == 64 and P.chunks_per_page(8) == 32
    # 3-bit pages leave 65536 - 85*768 = 256 bytes unused
    assert 65536 - 85 * L.chunk_bytes(3) == 256
    # pages needed = ceil(chunks / per page)
    H, F = 2048, 768
    n = L.n_chunks(H, F)
    assert n == 2304
    assert P.pages_needed(3, H, F) == 28 and P.pages_needed(4, H, F) == 36
    assert P.pages_needed(8, H, F) == 72


def test_allocator_hand_example():
    H, F = 128, 1280  # n_chunks = 3 * (1280/16) * (128/128) = 240
    assert L.n_chunks(H, F) == 240
    # pages: b=3 -> ceil(240/85)=3, b=4 -> ceil(240/64)=4, b=8 -> ceil(240/32)=8
    a = P.PageAllocator(pool_pages=20, E=3, H=H, F=F)
    changed = a.place(np.array([3, 4, 3], np.uint8))
    assert changed == [0, 1, 2]
    assert a.pages == [[0, 1, 2], [3, 4, 5, 6], [7, 8, 9]]
    t = a.table()
    assert list(t.first) == [0, 3, 7] and list(t.n_pages) == [3, 4, 3]
    assert list(t.page_idx) == list(range(10))
    # expert 1 drops to 3 bits, expert 2 rises to 8: both release, then both take
    # lowest-first: e1 gets 3,4,5; e2 gets 6,7,8,9,10,11,12,13
    changed = a.repage(np.array([3, 3, 8], np.uint8))
    assert changed == [1, 2]
    assert a.pages == [[0, 1, 2], [3, 4, 5], [6, 7, 8, 9, 10, 11, 12, 13]]
    assert a.used() == 14 and a.used() + int(a.free.sum()) == 20
    # pool too small for everything at 8 bits: nothing changes
    before = [list(p) for p in a.pages]
    with pytest.raises(P.PoolExhausted):
        a.repage(np.array([8, 8, 8], np.uint8))
    assert a.pages == before and list(a.bits) == [3, 3, 8]


@pytest.mark.parametrize("seed", range(4))
def test_allocator_invariants_random(seed):
    rng = np.random.default_rng(seed)
    E, H, F = 16, 256, 512
    a = P.PageAllocator(pool_pages=16 * P.pages_needed(8, H, F), E=E, H=H, F=F)
    bits = rng.choice([3, 4, 8], size=E).astype(np.uint8)
    a.place(bits)
    for _ in range(6):
        old_pages = [list(p) for p in a.pages]
        old_bits = a.bits.copy()
        new = rng.choice([3, 4, 8], size=E).astype(np.uint8)
        changed = a.repage(new)
        allp = [p for e in range(E) for p in a.pages[e]]
        assert len(allp) == len(set(allp))                       # disjoint
        assert a.used() == len(allp) and a.used() + a.free.sum() == a.pool_pages
        for e in range(E):
            assert len(a.pages[e]) == P.pages_needed(int(new[e]), H, F)
            if new[e] == old_bits[e]:
                assert e not in changed and a.pages[e] == old_pages[e]  # unchanged keep pages
            else:
                assert e in changed


def test_place_and_gather_stream():
    b, H, F = 4, 128, 128
    nch = L.n_chunks(H, F)
    stream = np.random.default_rng(0).integers(0, 256, size=(nch, L.chunk_bytes(b)), dtype=np.uint8)
    pool = np.zeros(4 * 65536, np.uint8)
    P.place_stream(pool, [2], stream, b)
    assert np.array_equal(P.gather_stream(pool, [2], nch, b), stream)
    assert np.all(pool[:2 * 65536] == 0)


def test_overlapped_repage_keeps_old_pages_until_commit():
    H, F = 256, 256
    E = 4
    need8 = P.pages_needed(8, H, F)
    need3 = P.pages_needed(3, H, F)
    A = P.PageAllocator(E * need8 + 2 * need3, E, H, F)
    A.place(np.array([8, 8, 8, 8], np.uint8))
    old = [list(x) for x in A.pages]
    changed = A.repage_overlapped(np.array([3, 8, 3, 8], np.uint8))
    assert changed == [0, 2]
    # unchanged experts keep their pages; new pages avoid every old page
    assert A.pages[1] == old[1] and A.pages[3] == old[3]
    in_use_before = set(p for x in old for p in x)
    assert not (set(A.pages[0]) | set(A.pages[2])) & in_use_before
    # lowest free pages first, ascending e: right after the 8-bit experts
    assert A.pages[0] == list(range(E * need8, E * need8 + need3))
    assert A.pages[2] == list(range(E * need8 + need3, E * need8 + 2 * need3))
    # old pages stay allocated until the commit
    assert A.used() == E * need8 + 2 * need3
    with pytest.raises(RuntimeError):
        A.repage_overlapped(np.array([3, 3, 3, 3], np.uint8))
    A.commit()
    assert A.used() == 2 * need8 + 2 * need3
    assert all(A.free[p] for p in old[0] + old[2])
    # after the commit the freed pages are reused, lowest first
    A.repage_overlapped(np.array([3, 3, 3, 8], np.uint8))
    assert A.pages[1] == list(range(need3))
    A.commit()


def test_overlapped_repage_is_transactional():
    H, F = 256, 256
    need8 = P.pages_needed(8, H, F)
    A = P.PageAllocator(2 * need8, 2, H, F)
    A.place(np.array([8, 8], np.uint8))
    t0 = A.table()
    with pytest.raises(P.PoolExhausted):
        A.repage_overlapped(np.array([4, 8], np.uint8))  # no free page for the new ones
    t1 = A.table()
    assert np.array_equal(t0.page_idx, t1.page_idx) and list(A.bits) == [8, 8]
    assert A.pending_release is None
