"""Token-to-expert bucketing.

PagedWeight, "Dynamic Paging": in a forward pass the router decides which
experts are needed; their pages are then fetched. The bucketing below groups
the routed (token, slot) assignments by expert so each expert's pages serve
all of its tokens at once.

Assignment a = t*k + j is token t's j-th routed expert ids[t, j].
* perm   -- the assignments sorted by expert id, stable (equal ids keep
            ascending a);
* offsets[E+1] -- exclusive prefix sum of the per-expert counts;
* inv[a] -- the position of a in perm.
Ids outside [0, E) are dropped: they appear in no bucket and inv = -1
(reading taken: the pages say nothing; an invalid id must not touch memory).
"""
from __future__ import annotations

import numpy as np


def route(ids, E: int):
    ids = np.asarray(ids, dtype=np.int64).ravel()
    valid = (ids >= 0) & (ids < E)
    a_valid = np.flatnonzero(valid)
    order = np.argsort(ids[a_valid], kind="stable")
    perm = a_valid[order].astype(np.int32)
    counts = np.bincount(ids[a_valid], minlength=E)
    offsets = np.zeros(E + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    inv = np.full(ids.size, -1, dtype=np.int32)
    inv[perm] = np.arange(perm.size, dtype=np.int32)
    return perm, offsets, inv
