"""Packed page format for 3-, 4- and 8-bit expert codes.

PagedWeight, "Dynamic Paging": expert weights are quantized and stored in
pages of varying bit-widths (8-, 4-, 3-bit). The page does not give a byte
format; this module is the project's own definition, written out plainly.

Terms. A matrix [R x K] (row = output feature, K contiguous) at bit width b
needs R % 16 == 0 and K % 128 == 0.
* block   -- 128 consecutive codes of one row, k in [128 j, 128 j + 128);
             16*b bytes.
* quarter -- 32 consecutive codes of a block, k = 128 j + 32 q + i', i' < 32;
             4*b bytes at byte offset 4*b*q of its block.
* chunk   -- 16 blocks: rows 16*tau .. 16*tau + 15, block column j; 256*b bytes.
             Block of row 16*tau + rho sits at byte offset 16*b*rho.
             Chunks of a matrix run tau-major: chunk index c = tau*(K/128) + j.
* expert stream -- the chunks of W1 (gate, [F x H]) and W3 (up, [F x H])
             interleaved, chunk 2c = W1's chunk c and 2c+1 = W3's chunk c, then
             the chunks of W2 (down, [H x F]). A gate row's block and the up
             row's block for the same feature and K range are thus adjacent, and
             so are a tile's consecutive block columns of both.

Inside a quarter the 32 codes c'_0 .. c'_31 are b little-endian 32-bit words:
* b = 8: word w (0..7) holds c'_{4w+i} at bit 16*(i&1) + 8*(i>>1), i = 0..3.
* b = 4: word w (0..3) holds c'_{8w+i} at bit 16*(i&1) + 4*(i>>1), i = 0..7.
* b = 3: word v (0..2) holds c'_{10v+i} at bit 16*(i&1) + 3*(i>>1), i = 0..9;
         bit n (n = 0,1,2) of c'_30 is bit 15 of word n and bit n of c'_31 is
         bit 31 of word n.
* b = 1: word 0 holds c'_i at bit 16*(i&1) + (i>>1), i = 0..31 (not a width
         of the main format: the one-bit layer of the prefix-compatible store,
         oracle/prefix.py, uses it).
In every width the pair (c'_{2m}, c'_{2m+1}) sits at the same position of the
low and the high 16-bit half of one word (the spare pair of b = 3 excepted).

Codes are offset binary u = k + 2^(b-1).
"""
from __future__ import annotations

import numpy as np

ROWS_PER_CHUNK = 16
CODES_PER_BLOCK = 128
CODES_PER_QUARTER = 32


def block_bytes(b: int) -> int:
    return 16 * b


def chunk_bytes(b: int) -> int:
    return ROWS_PER_CHUNK * block_bytes(b)


def _shifts(b: int) -> np.ndarray:
    if b == 1:
        return np.array([16 * (i & 1) + (i >> 1) for i in range(32)], dtype=np.uint32)
    if b == 8:
        return np.array([16 * (i & 1) + 8 * (i >> 1) for i in range(4)], dtype=np.uint32)
    if b == 4:
        return np.array([16 * (i & 1) + 4 * (i >> 1) for i in range(8)], dtype=np.uint32)
    if b == 3:
        return np.array([16 * (i & 1) + 3 * (i >> 1) for i in range(10)], dtype=np.uint32)
    raise ValueError(f"bit width {b} not in (1, 3, 4, 8)")


def pack_quarters(u: np.ndarray, b: int) -> np.ndarray:
    """u: uint [..., 32] offset codes -> uint32 words [..., b]."""
    u = np.asarray(u, dtype=np.uint32)
    assert u.shape[-1] == CODES_PER_QUARTER
    lead = u.shape[:-1]
    mask = np.uint32((1 << b) - 1)
    if np.any(u > mask):
        raise ValueError("code out of range for bit width")
    sh = _shifts(b)
    if b in (1, 4, 8):
        per = 32 // b
        g = u.reshape(lead + (b, per))
        words = np.zeros(lead + (b,), dtype=np.uint32)
        for i in range(per):
            words |= g[..., i] << sh[i]
        return words
    # b == 3
    g = u[..., :30].reshape(lead + (3, 10))
    words = np.zeros(lead + (3,), dtype=np.uint32)
    for i in range(10):
        words |= g[..., i] << sh[i]
    for n in range(3):
        words[..., n] |= ((u[..., 30] >> np.uint32(n)) & np.uint32(1)) << np.uint32(15)
        words[..., n] |= ((u[..., 31] >> np.uint32(n)) & np.uint32(1)) << np.uint32(31)
    return words


def unpack_quarters(words: np.ndarray, b: int) -> np.ndarray:
    """uint32 words [..., b] -> uint32 offset codes [..., 32]."""
    words = np.asarray(words, dtype=np.uint32)
    assert words.shape[-1] == b
    lead = words.shape[:-1]
    mask = np.uint32((1 << b) - 1)
    sh = _shifts(b)
    u = np.zeros(lead + (CODES_PER_QUARTER,), dtype=np.uint32)
    if b in (1, 4, 8):
        per = 32 // b
        for w in range(b):
            for i in range(per):
                u[..., per * w + i] = (words[..., w] >> sh[i]) & mask
        return u
    for v in range(3):
        for i in range(10):
            u[..., 10 * v + i] = (words[..., v] >> sh[i]) & mask
    c30 = np.zeros(lead, dtype=np.uint32)
    c31 = np.zeros(lead, dtype=np.uint32)
    for n in range(3):
        c30 |= ((words[..., n] >> np.uint32(15)) & np.uint32(1)) << np.uint32(n)
        c31 |= ((words[..., n] >> np.uint32(31)) & np.uint32(1)) << np.uint32(n)
    u[..., 30] = c30
    u[..., 31] = c31
    return u


def pack_matrix(u: np.ndarray, b: int, tile_batch: int = 64) -> np.ndarray:
    """Offset codes [R, K] -> chunk stream uint8 [R/16 * K/128, 256*b], chunk order tau-major."""
    u = np.asarray(u)
    R, K = u.shape
    if R % ROWS_PER_CHUNK or K % CODES_PER_BLOCK:
        raise ValueError("matrix needs R % 16 == 0 and K % 128 == 0")
    nt, nj = R // ROWS_PER_CHUNK, K // CODES_PER_BLOCK
    out = np.empty((nt, nj, chunk_bytes(b)), dtype=np.uint8)
    for t0 in range(0, nt, tile_batch):
        t1 = min(nt, t0 + tile_batch)
        sub = u[t0 * 16:t1 * 16].astype(np.uint32)
        # [tiles, rho, j, quarter, i'] -> [tiles, j, rho, quarter, i']
        sub = sub.reshape(t1 - t0, ROWS_PER_CHUNK, nj, 4, CODES_PER_QUARTER)
        sub = sub.transpose(0, 2, 1, 3, 4)
        words = pack_quarters(sub, b)                       # [tiles, j, rho, q, b]
        out[t0:t1] = words.astype("<u4").reshape(t1 - t0, nj, -1).view(np.uint8)
    return out.reshape(nt * nj, chunk_bytes(b))


def unpack_matrix(stream: np.ndarray, R: int, K: int, b: int) -> np.ndarray:
    """Inverse of pack_matrix: chunk stream -> offset codes [R, K]."""
    nt, nj = R // ROWS_PER_CHUNK, K // CODES_PER_BLOCK
    words = np.ascontiguousarray(stream).reshape(nt, nj, -1).view("<u4")
    words = words.reshape(nt, nj, ROWS_PER_CHUNK, 4, b)
    u = unpack_quarters(words, b)                           # [tiles, j, rho, q, 32]
    return u.transpose(0, 2, 1, 3, 4).reshape(R, K)


def n_chunks(H: int, F: int) -> int:
    """Chunks in one expert stream: W1 and W3 [F x H], W2 [H x F]."""
    return 3 * (F // ROWS_PER_CHUNK) * (H // CODES_PER_BLOCK)


def expert_stream(u1: np.ndarray, u3: np.ndarray, u2: np.ndarray, b: int) -> np.ndarray:
    """Chunk stream of one expert: W1 and W3 chunk by chunk (W1 chunk c at 2c,
    W3 chunk c at 2c + 1), then W2 with each pair of row tiles interleaved by
    block column (tile 2v's chunk j at 2(v nj + j), tile 2v+1's at
    2(v nj + j) + 1 after the gate/up chunks). uint8 [n_chunks, 256*b]."""
    g1, g3 = pack_matrix(u1, b), pack_matrix(u3, b)
    gu = np.stack([g1, g3], axis=1).reshape(2 * g1.shape[0], chunk_bytes(b))
    R2, K2 = np.asarray(u2).shape
    nt2, nj2 = R2 // ROWS_PER_CHUNK, K2 // CODES_PER_BLOCK
    if nt2 % 2:
        raise ValueError("W2 needs an even number of 16-row tiles (H % 32 == 0)")
    g2 = pack_matrix(u2, b).reshape(nt2 // 2, 2, nj2, chunk_bytes(b))
    g2 = g2.transpose(0, 2, 1, 3).reshape(nt2 * nj2, chunk_bytes(b))
    return np.concatenate([gu, g2])
