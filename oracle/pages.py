"""Page allocator and page table (simulation).

PagedWeight, "Dynamic Paging": GPU memory is divided into pages and experts
are stored in pages of one bit width; "Implementation Details", memory
management: a page table maps expert IDs to physical page addresses, and the
scheduler re-sizes experts' pages as KV-cache occupancy changes; "Code
Illustration": an expert's page_size is set by the allocator.

Readings taken where the pages leave the step open:
* Physical pages have one fixed size P (default 64 KiB). A page holds whole
  chunks (16 rows x 128 codes) of one expert at one bit width:
  chunks_per_page(b) = floor(P / (256 b)) = 85 / 64 / 32 at b = 3 / 4 / 8.
  An expert's "page size" is then n_pages * P.
* Allocation is deterministic: each request takes the lowest-numbered free
  pages, one by one (not necessarily contiguous).
* Initial placement: experts in ascending order.
* Repage: the experts whose width changed release their pages (ascending e),
  then the same experts receive new pages (ascending e). Experts whose width
  is unchanged keep their pages. If the pool cannot satisfy the request,
  nothing changes (transactional).
* Page table: per expert (bits, first, n_pages); first indexes one compact
  page-index array that lists each expert's pages in stream order, experts
  in ascending order.
* Overlapped repage (the scheduler changes precision while decode goes on):
  the changed experts keep their old pages readable until a commit, so their
  new pages come from the pages free at the call (lowest index first,
  ascending e); the old pages return to the pool at the commit. Transactional
  as well; one overlapped repage at a time.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

from .layout import chunk_bytes, n_chunks

DEFAULT_PAGE_BYTES = 1 << 16


class PoolExhausted(RuntimeError):
    """Not enough free pages; the allocator state is unchanged."""


def chunks_per_page(b: int, page_bytes: int = DEFAULT_PAGE_BYTES) -> int:
    return page_bytes // chunk_bytes(b)


def pages_needed(b: int, H: int, F: int, page_bytes: int = DEFAULT_PAGE_BYTES) -> int:
    return math.ceil(n_chunks(H, F) / chunks_per_page(b, page_bytes))


@dataclasses.dataclass
class PageTable:
    bits: np.ndarray        # uint8 [E]
    first: np.ndarray       # uint32 [E]
    n_pages: np.ndarray     # uint32 [E]
    page_idx: np.ndarray    # uint32 [sum n_pages]


class PageAllocator:
    """Bitmap pool with lowest-index-first allocation."""

    def __init__(self, pool_pages: int, E: int, H: int, F: int,
                 page_bytes: int = DEFAULT_PAGE_BYTES):
        self.pool_pages = pool_pages
        self.E, self.H, self.F = E, H, F
        self.page_bytes = page_bytes
        self.free = np.ones(pool_pages, dtype=bool)
        self.pages: list[list[int]] = [[] for _ in range(E)]
        self.bits = np.zeros(E, dtype=np.uint8)
        self.pending_release: list[int] | None = None

    def _take(self, free: np.ndarray, n: int) -> list[int]:
        idx = np.flatnonzero(free)[:n]
        if len(idx) < n:
            raise PoolExhausted(f"need {n} pages, {len(idx)} free")
        free[idx] = False
        return [int(i) for i in idx]

    def place(self, bits) -> list[int]:
        """Initial placement (or re-placement) for the given widths; returns changed experts."""
        return self.repage(bits)

    def repage(self, new_bits) -> list[int]:
        new_bits = np.asarray(new_bits, dtype=np.uint8)
        changed = [e for e in range(self.E) if int(new_bits[e]) != int(self.bits[e])]
        free = self.free.copy()
        pages = [list(p) for p in self.pages]
        for e in changed:
            free[pages[e]] = True
            pages[e] = []
        for e in changed:
            n = pages_needed(int(new_bits[e]), self.H, self.F, self.page_bytes)
            pages[e] = self._take(free, n)
        self.free = free
        self.pages = pages
        self.bits = new_bits.copy()
        return changed

    def repage_overlapped(self, new_bits) -> list[int]:
        """Repage while the old pages stay in use: new pages for the changed
        experts from the currently free pages; the old ones are released by
        commit(). Returns the changed experts (the table shows the new pages)."""
        if self.pending_release is not None:
            raise RuntimeError("an overlapped repage is pending: commit it first")
        new_bits = np.asarray(new_bits, dtype=np.uint8)
        changed = [e for e in range(self.E) if int(new_bits[e]) != int(self.bits[e])]
        free = self.free.copy()
        pages = [list(p) for p in self.pages]
        released: list[int] = []
        for e in changed:
            n = pages_needed(int(new_bits[e]), self.H, self.F, self.page_bytes)
            new_pages = self._take(free, n)
            released.extend(pages[e])
            pages[e] = new_pages
        self.free = free
        self.pages = pages
        self.bits = new_bits.copy()
        self.pending_release = released
        return changed

    def commit(self) -> None:
        """Release the old pages of the last overlapped repage."""
        if self.pending_release:
            self.free[self.pending_release] = True
        self.pending_release = None

    def table(self) -> PageTable:
        first = np.zeros(self.E, dtype=np.uint32)
        n = np.zeros(self.E, dtype=np.uint32)
        idx = []
        for e in range(self.E):
            first[e] = len(idx)
            n[e] = len(self.pages[e])
            idx.extend(self.pages[e])
        return PageTable(self.bits.copy(), first, n, np.asarray(idx, dtype=np.uint32))

    def used(self) -> int:
        return int((~self.free).sum())


def place_stream(pool: np.ndarray, pages: list[int], stream: np.ndarray, b: int,
                 page_bytes: int = DEFAULT_PAGE_BYTES) -> None:
    """Write one expert's chunk stream into a byte image of the pool through its pages."""
    cpp = chunks_per_page(b, page_bytes)
    cb = chunk_bytes(b)
    for c in range(stream.shape[0]):
        page = pages[c // cpp]
        off = page * page_bytes + (c % cpp) * cb
        pool[off:off + cb] = stream[c]


def gather_stream(pool: np.ndarray, pages: list[int], nchunks: int, b: int,
                  page_bytes: int = DEFAULT_PAGE_BYTES) -> np.ndarray:
    """Read one expert's chunk stream back out of a pool image through its pages."""
    cpp = chunks_per_page(b, page_bytes)
    cb = chunk_bytes(b)
    out = np.empty((nchunks, cb), dtype=np.uint8)
    for c in range(nchunks):
        page = pages[c // cpp]
        off = page * page_bytes + (c % cpp) * cb
        out[c] = pool[off:off + cb]
    return out
