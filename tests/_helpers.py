"""Shared pieces of the GPU parity tests: oracle-side expected values (oracle/
and synth only) and the FFN tolerance check."""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import synth
from oracle import ffn as of
from oracle import layout as ol
from oracle import quantize as oq

# FFN tolerance for bf16 activations with fp32 accumulation (stated for the
# method's routed expert FFN): relative Frobenius error and max abs error
# relative to the oracle's largest magnitude.
REL_FRO = 5e-3
MAX_ABS_REL = 2e-2


def check_ffn(got: np.ndarray, ref: np.ndarray):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got))
    nref = np.linalg.norm(ref)
    if nref == 0.0:
        assert np.all(got == 0.0)
        return 0.0, 0.0
    rel = np.linalg.norm(got - ref) / nref
    mx = np.abs(got - ref).max() / np.abs(ref).max()
    assert rel <= REL_FRO, f"rel Frobenius {rel:.3e} > {REL_FRO}"
    assert mx <= MAX_ABS_REL, f"max abs {mx:.3e} > {MAX_ABS_REL} * max|ref|"
    return rel, mx


class OracleExpert:
    """Oracle view of one expert: absmax, scale, codes, packed stream, dequantized mats."""

    def __init__(self, master_fp16: np.ndarray, H: int, F: int, b: int):
        self.H, self.F, self.b = H, F, b
        self.m, self.s, self.k = oq.quantize_expert(master_fp16, b)

    def stream(self) -> np.ndarray:
        H, F, b = self.H, self.F, self.b
        u = oq.offset_codes(self.k, b)
        return ol.expert_stream(u[:F * H].reshape(F, H), u[F * H:2 * F * H].reshape(F, H),
                                u[2 * F * H:].reshape(H, F), b).reshape(-1)

    def mats(self):
        H, F = self.H, self.F
        d = oq.dequantize(self.k, self.s)
        return (d[:F * H].reshape(F, H), d[F * H:2 * F * H].reshape(F, H),
                d[2 * F * H:].reshape(H, F))


# every 16-bit pattern as an fp16 value, and which of them are finite
_FP16_ALL = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16).view(np.float16)
_FP16_FINITE = np.isfinite(_FP16_ALL)


class OracleExpertByValue:
    """The oracle's view of one expert -- absmax, scale, packed stream,
    dequantized matrices -- with the per-weight steps evaluated once per
    distinct fp16 value, so that experts of tens of millions of weights can be
    checked in full.

    The oracle's encode() and dequantize() act on each weight alone (the code
    of w depends only on w, s and b), so mapping every weight through a
    65,536-entry table of encode() over all fp16 bit patterns gives exactly
    the array encode() would return; absmax() over the distinct values that
    occur equals absmax() over the array (repeats do not change a maximum,
    and a NaN or infinity among them still raises). The packing is the
    oracle's expert_stream() on the gathered codes. tests/test_oracle_by_value.py
    checks all of this against OracleExpert on whole experts."""

    def __init__(self, master_fp16: np.ndarray, H: int, F: int, b: int):
        master = np.ascontiguousarray(master_fp16)
        assert master.dtype == np.float16 and master.size == 3 * H * F
        self.H, self.F, self.b = H, F, b
        self._bits = master.view(np.uint16)
        seen = np.bincount(self._bits, minlength=1 << 16)
        present = np.flatnonzero(seen).astype(np.uint16).view(np.float16)
        self.m = oq.absmax(present)
        self.s = oq.scale(self.m, b)
        k_tab = np.zeros(1 << 16, dtype=np.int64)
        k_tab[_FP16_FINITE] = oq.encode(_FP16_ALL[_FP16_FINITE], self.s, b)
        self._k_tab = k_tab

    def codes(self) -> np.ndarray:
        """k for every weight (int64)."""
        return self._k_tab[self._bits]

    def stream(self) -> np.ndarray:
        H, F, b = self.H, self.F, self.b
        u = oq.offset_codes(self._k_tab, b).astype(np.uint8)[self._bits]
        return ol.expert_stream(u[:F * H].reshape(F, H), u[F * H:2 * F * H].reshape(F, H),
                                u[2 * F * H:].reshape(H, F), b).reshape(-1)

    def mats(self):
        H, F = self.H, self.F
        d = oq.dequantize(self._k_tab, self.s)[self._bits]
        return (d[:F * H].reshape(F, H), d[F * H:2 * F * H].reshape(F, H),
                d[2 * F * H:].reshape(H, F))


def oracle_threads() -> int:
    return max(1, min(32, len(os.sched_getaffinity(0))))


def check_experts_in_full(ctx, masters_dev, bits, H: int, F: int, experts=None):
    """Absmax, scale and the whole packed stream (read back through the device
    page table) of each listed expert, bit-exact against the oracle. The
    device reads run in this thread; the oracle's work runs in a thread pool
    (NumPy releases the interpreter lock in its array loops)."""
    experts = range(len(masters_dev)) if experts is None else experts
    scales, absmax = ctx.scales()

    def one(e, master, got):
        ox = OracleExpertByValue(master, H, F, int(bits[e]))
        ref = ox.stream()
        bad = None if np.array_equal(got, ref) else np.flatnonzero(got != ref)[:8]
        return e, ox.m, ox.s, got.size == ref.size, bad

    n_workers = oracle_threads()
    results, pending = [], []
    with ThreadPoolExecutor(n_workers) as pool:
        for e in experts:
            e = int(e)
            master = masters_dev[e].cpu().numpy()
            got = ctx.expert_stream(e)
            pending.append(pool.submit(one, e, master, got))
            if len(pending) >= 2 * n_workers:
                results.append(pending.pop(0).result())
        results += [f.result() for f in pending]
    for e, m, s, same_size, bad in results:
        assert absmax[e] == np.float32(m), (e, absmax[e], m)
        assert scales[e] == s, (e, scales[e], s)
        assert same_size, e
        assert bad is None, f"expert {e} at {int(bits[e])} bits: bytes {bad} differ"
    return len(results)


def workload_masters_cpu(wl, e) -> np.ndarray:
    return synth.expert_weights(wl, e).numpy()


def workload_masters_gpu(wl, device="cuda"):
    out = []
    for e in range(wl.E):
        t = torch.empty(wl.W_e, dtype=torch.float16, device=device)
        synth.fill_expert_weights(wl, e, t)
        out.append(t)
    return out


def oracle_moe(x_bf16: torch.Tensor, ids: np.ndarray, w: np.ndarray, mats_of, E: int,
               tokens=None) -> np.ndarray:
    return of.moe_ffn(x_bf16.double().cpu().numpy(), ids, w, mats_of, E, tokens=tokens)


def oracle_moe_parallel(x_bf16: torch.Tensor, ids: np.ndarray, w: np.ndarray, mats_of,
                        E: int, tokens=None, workers: int | None = None) -> np.ndarray:
    """oracle moe_ffn split by expert over a thread pool: each call sees the
    ids of its share of the experts (the others marked -1, which the oracle
    drops), and the layer output is the sum of the shares (the combine is a
    sum over slots, so the shares add up to the whole layer; only the order of
    the float64 additions differs)."""
    x = x_bf16.double().cpu().numpy()
    ids = np.asarray(ids)
    used = np.unique(ids[(ids >= 0) & (ids < E)])
    if tokens is not None:
        sub = ids[np.asarray(tokens)]
        used = np.unique(sub[(sub >= 0) & (sub < E)])
    n = workers or max(1, min(8, oracle_threads()))
    shares = [used[i::n] for i in range(n) if used[i::n].size]

    def part(experts):
        mask = np.isin(ids, experts)
        return of.moe_ffn(x, np.where(mask, ids, -1), w, mats_of, E, tokens=tokens)

    with ThreadPoolExecutor(len(shares) or 1) as pool:
        outs = list(pool.map(part, shares))
    if not outs:
        return of.moe_ffn(x, ids, w, mats_of, E, tokens=tokens)
    return np.sum(outs, axis=0)


def check_page_table(ctx, alloc, bits):
    """The device page table (widths, first page-index entry, page counts and
    the page-index array) equals the oracle allocator's."""
    pte, pidx = ctx.page_table()
    table = alloc.table()
    assert np.array_equal(pte["bits"], np.asarray(bits, np.uint8))
    assert np.array_equal(pte["first"], table.first)
    assert np.array_equal(pte["n_pages"], table.n_pages)
    assert np.array_equal(pidx, table.page_idx)
