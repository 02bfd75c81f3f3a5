"""Prefix-compatible quantizer and layered page store (a variant of the main
format), float64 / exact integers.

What it follows: the bitplane idea of storing a high-precision code so that
every lower precision is a prefix of it, so that a precision change only adds
or drops the low-order bits instead of re-encoding the expert; PagedWeight,
"Dynamic Paging" / "Implementation Details": experts live in pages, and the
scheduler lowers or raises their precision as KV-cache occupancy changes.
The main format's symmetric grid (s = m / (2^(b-1) - 1)) is not nested
across widths, so this variant uses a nested grid.

Readings taken where the pages leave the step open:
* Grid: 2^b uniform bins over [-m, m] (m = max |w| of the expert), the value
  of a bin its centre. The 8-bit code is u8 = clamp(floor(128 w / m) + 128,
  0, 255), taken exactly; the b-bit code is its top b bits, u_b = u8 >> (8 - b);
  w^_b = (m / 2^b) (2 u_b + 1 - 2^b). m = 0 gives u8 = 128 and w^ = 0.
  |w - w^_b| <= m / 2^b (half a bin).
* Layers: A = u8 >> 5 (3 bits), B = bit 4 of u8, C = u8 & 15. A 3-bit expert
  stores A, a 4-bit one A and B, an 8-bit one A, B and C:
  u_4 = 2 u_3 + B, u_8 = 16 u_4 + C.
* Layer streams: each layer of an expert is a chunk stream in the main
  format's layout (oracle/layout.py) at the layer's width (A 3 bits, B 1
  bit, C 4 bits): the layer's codes of W1, W3 [F x H] and W2 [H x F] packed
  as layout.expert_stream packs an expert's codes, so that chunk n of every
  layer covers the same 16 rows x 128 codes (H and F multiples of 128). The
  pages fix no byte format; this one lets a forward pass read the layers of
  a chunk side by side, with the main format's in-register unpack.
* Pages: every layer of every expert has its own pages holding whole chunks
  (floor(P / chunk bytes) a page, 256 * layer bits bytes a chunk).
  Placement takes the lowest free pages, experts ascending, layers A, B, C.
  A width change drops the removed layers' pages (no encode at all) or adds
  pages for the new layers and encodes only those; the changed experts
  release first (ascending e), then allocate (ascending e); unchanged
  layers keep their pages; on shortage nothing changes.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

from oracle import layout

LAYER_BITS = {"A": 3, "B": 1, "C": 4}


def layers_of(b: int) -> tuple[str, ...]:
    return {3: ("A",), 4: ("A", "B"), 8: ("A", "B", "C")}[b]


def prefix_codes(master_fp16) -> tuple[float, np.ndarray]:
    """(m, u8) for one expert's flat fp16 master; u8 int64 in [0, 255].
    Exact: every fp16 value is an integer multiple of 2^-24, so
    floor(128 w / m) is an integer floor division."""
    w = np.asarray(master_fp16)
    assert w.dtype == np.float16
    if w.size and not np.isfinite(w).all():
        raise ValueError("master contains NaN or Inf")
    wd = w.astype(np.float64)
    m = float(np.max(np.abs(wd))) if w.size else 0.0
    if m == 0.0:
        return m, np.full(w.shape, 128, dtype=np.int64)
    wi = (wd * 2.0 ** 24).astype(np.int64)   # exact
    mi = int(m * 2.0 ** 24)
    u8 = (128 * wi) // mi + 128               # floor division of exact integers
    return m, np.clip(u8, 0, 255)


def code_of_width(u8: np.ndarray, b: int) -> np.ndarray:
    return np.asarray(u8, dtype=np.int64) >> (8 - b)


def dequantize(m: float, u_b: np.ndarray, b: int) -> np.ndarray:
    """w^_b = (m / 2^b)(2 u_b + 1 - 2^b), float64 (exact)."""
    return (m / float(1 << b)) * (2.0 * np.asarray(u_b, dtype=np.float64) + 1.0 - float(1 << b))


def layer_values(u8: np.ndarray, layer: str) -> np.ndarray:
    u8 = np.asarray(u8, dtype=np.int64)
    return {"A": u8 >> 5, "B": (u8 >> 4) & 1, "C": u8 & 15}[layer]


def _mats(flat: np.ndarray, H: int, F: int):
    flat = np.asarray(flat)
    return (flat[:F * H].reshape(F, H), flat[F * H:2 * F * H].reshape(F, H),
            flat[2 * F * H:].reshape(H, F))


def layer_stream(u8_flat: np.ndarray, layer: str, H: int, F: int) -> np.ndarray:
    """Layer `layer` of one expert (u8_flat: W1 | W3 | W2 row-major) as its
    chunk stream, uint8 [n_chunks, 256 * bits]."""
    v1, v3, v2 = _mats(layer_values(u8_flat, layer).astype(np.uint32), H, F)
    return layout.expert_stream(v1, v3, v2, LAYER_BITS[layer])


def layer_codes(stream: np.ndarray, layer: str, H: int, F: int) -> np.ndarray:
    """Inverse of layer_stream: the layer's codes, W1 | W3 | W2 row-major."""
    b = LAYER_BITS[layer]
    cb = layout.chunk_bytes(b)
    s = np.asarray(stream, dtype=np.uint8).reshape(-1, cb)
    nc1 = (F // 16) * (H // 128)
    gu = s[:2 * nc1].reshape(nc1, 2, cb)
    u1 = layout.unpack_matrix(gu[:, 0], F, H, b)
    u3 = layout.unpack_matrix(gu[:, 1], F, H, b)
    nt2, nj2 = H // 16, F // 128
    g2 = s[2 * nc1:].reshape(nt2 // 2, nj2, 2, cb).transpose(0, 2, 1, 3).reshape(-1, cb)
    u2 = layout.unpack_matrix(g2, H, F, b)
    return np.concatenate([u1.reshape(-1), u3.reshape(-1), u2.reshape(-1)]).astype(np.int64)


def chunk_bytes(layer: str) -> int:
    return layout.chunk_bytes(LAYER_BITS[layer])


def chunks_per_page(layer: str, page_bytes: int) -> int:
    return page_bytes // chunk_bytes(layer)


def layer_pages(layer: str, H: int, F: int, page_bytes: int) -> int:
    return math.ceil(layout.n_chunks(H, F) / chunks_per_page(layer, page_bytes))


class PoolExhausted(RuntimeError):
    """Not enough free pages; nothing changed."""


@dataclasses.dataclass
class LayeredPages:
    """Page bookkeeping of the layered store: pages[e][layer] lists pages."""
    n_pages: int
    E: int
    H: int
    F: int
    page_bytes: int

    def __post_init__(self):
        self.free = np.ones(self.n_pages, dtype=bool)
        self.pages = [dict() for _ in range(self.E)]
        self.bits = np.zeros(self.E, dtype=np.uint8)

    def _take(self, free, n):
        idx = np.flatnonzero(free)[:n]
        if len(idx) < n:
            raise PoolExhausted(f"need {n} pages, {len(idx)} free")
        free[idx] = False
        return [int(i) for i in idx]

    def place(self, bits):
        """Initial placement; returns {e: layers encoded}."""
        free = self.free.copy()
        pages = [dict() for _ in range(self.E)]
        for e in range(self.E):
            for L in layers_of(int(bits[e])):
                pages[e][L] = self._take(free, layer_pages(L, self.H, self.F, self.page_bytes))
        self.free, self.pages = free, pages
        self.bits = np.asarray(bits, dtype=np.uint8).copy()
        return {e: list(layers_of(int(bits[e]))) for e in range(self.E)}

    def repage(self, new_bits):
        """Width change; returns {e: layers to encode} (only added layers)."""
        new_bits = np.asarray(new_bits, dtype=np.uint8)
        free = self.free.copy()
        pages = [dict(p) for p in self.pages]
        changed = [e for e in range(self.E) if int(new_bits[e]) != int(self.bits[e])]
        for e in changed:  # release dropped layers, ascending e
            keep = set(layers_of(int(new_bits[e])))
            for L in list(pages[e]):
                if L not in keep:
                    free[pages[e][L]] = True
                    del pages[e][L]
        encode = {}
        for e in changed:  # allocate added layers, ascending e, layers in order
            added = [L for L in layers_of(int(new_bits[e])) if L not in pages[e]]
            for L in added:
                pages[e][L] = self._take(free, layer_pages(L, self.H, self.F, self.page_bytes))
            if added:
                encode[e] = added
        self.free, self.pages = free, pages
        self.bits = new_bits.copy()
        return encode

    def table(self):
        """(first[E], n_pages[E], page_idx): an expert's pages in layer order."""
        first = np.zeros(self.E, dtype=np.uint32)
        n = np.zeros(self.E, dtype=np.uint32)
        idx = []
        for e in range(self.E):
            first[e] = len(idx)
            for L in ("A", "B", "C"):
                if L in self.pages[e]:
                    idx.extend(self.pages[e][L])
            n[e] = len(idx) - first[e]
        return first, n, np.asarray(idx, dtype=np.uint32)


def repage_bytes(encode: dict, W_e: int) -> int:
    """Bytes a repage moves: the master read once per expert that encodes,
    plus the added layers written."""
    total = 0
    for e, layers in encode.items():
        total += 2 * W_e + sum(LAYER_BITS[L] * W_e // 8 for L in layers)
    return total


def expert_mats(master_fp16, H: int, F: int, b: int):
    """Dequantized (W1^, W3^, W2^) of one expert at b bits, float64."""
    m, u8 = prefix_codes(master_fp16)
    d = dequantize(m, code_of_width(u8, b), b)
    return (d[:F * H].reshape(F, H), d[F * H:2 * F * H].reshape(F, H),
            d[2 * F * H:].reshape(H, F))
