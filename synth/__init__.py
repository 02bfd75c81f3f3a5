"""Seeded synthetic inputs for the mixed-precision MoE expert path.

This module is the one piece of code that both sides use: the float64 oracle
(through the tests) and the CUDA path (through the tests and the benchmark).
It holds none of the method's arithmetic -- no absmax, no scale, no rounding
to codes, no packing, no FFN. It only draws inputs:

* fp16 master weights distributed as fp16(N(0, sigma)), optionally with
  outliers, from a counter-based integer generator, so that any single
  element of any expert can be regenerated on any device and both sides see
  bit-identical values (the GPU side draws on the device, the oracle on the
  host, from the same integer recipe);
* bf16 activations distributed as bf16(N(0, 1)), drawn the same way;
* router logits, top-k expert ids and softmax-renormalised top-k weights;
* expert importances p_e (Dirichlet or Zipf);
* the five workload shapes, their budgets and the dynamic-repaging schedule.

Integer generator: element i of stream (seed, stream) is
``u = lowbias32((i * 0x9E3779B1 mod 2^32) ^ key)`` with ``key`` derived from
(seed, stream); lowbias32 is the 32-bit integer finaliser published by
C. Wellons ("hash-prospector", xorshift-multiply, constants 0x7feb352d and
0x846ca68b). ``u`` selects a value by inverse CDF over every finite fp16 (or
bf16) value, with interval probabilities computed in float64 from the normal
CDF, so the draw follows the *rounded* normal distribution up to 2^-32.

Seeds follow ``1000 * cfg + purpose`` (0 weights, 1 outliers, 2 importance,
3 logits, 4 activations, 5 schedule); the stream id of an expert's weights
is its expert index.
"""
from __future__ import annotations

import dataclasses
import functools
import math

import numpy as np
import torch

MASK32 = 0xFFFFFFFF

PURPOSE_WEIGHTS = 0
PURPOSE_OUTLIERS = 1
PURPOSE_IMPORTANCE = 2
PURPOSE_LOGITS = 3
PURPOSE_ACTIVATIONS = 4
PURPOSE_SCHEDULE = 5


# ----------------------------------------------------------------------------
# counter-based integer generator
# ----------------------------------------------------------------------------
def _s32(c: int) -> int:
    """A uint32 constant as the int32 with the same bits."""
    c &= MASK32
    return c - (1 << 32) if c >= (1 << 31) else c


def _lowbias32(x: torch.Tensor) -> torch.Tensor:
    """lowbias32 on int32 tensors (bit patterns of uint32; products wrap mod 2^32)."""
    x = x ^ ((x >> 16) & 0xFFFF)
    x = x * _s32(0x7FEB352D)
    x = x ^ ((x >> 15) & 0x1FFFF)
    x = x * _s32(0x846CA68B)
    x = x ^ ((x >> 16) & 0xFFFF)
    return x


def _lowbias32_int(x: int) -> int:
    x &= MASK32
    x ^= x >> 16
    x = (x * 0x7FEB352D) & MASK32
    x ^= x >> 15
    x = (x * 0x846CA68B) & MASK32
    x ^= x >> 16
    return x


def _stream_key(seed: int, stream: int) -> int:
    k = _lowbias32_int((seed * 0x9E3779B1 + 0x27D4EB2F) & MASK32)
    return _lowbias32_int((k ^ (stream * 0x85EBCA77) ^ 0x165667B1) & MASK32)


def _u32_from_index(index: torch.Tensor, key: int) -> torch.Tensor:
    i = index.to(torch.int32) if index.dtype != torch.int32 else index
    x = (i * _s32(0x9E3779B1)) ^ _s32(key)
    return _lowbias32(x).to(torch.int64) & MASK32


def uniform_u32(seed: int, stream: int, start: int, count: int,
                device: torch.device | str = "cpu") -> torch.Tensor:
    """Elements [start, start+count) of integer stream (seed, stream): uint32 values in int64.

    Element i is lowbias32((i * 0x9E3779B1 mod 2^32) xor key(seed, stream))."""
    assert 0 <= start and start + count <= (1 << 32)
    idx = torch.arange(start, start + count, dtype=torch.int64, device=device)
    idx = torch.where(idx >= (1 << 31), idx - (1 << 32), idx).to(torch.int32)
    return _u32_from_index(idx, _stream_key(seed, stream))


def uniform_u32_at(seed: int, stream: int, index: torch.Tensor) -> torch.Tensor:
    """Elements at arbitrary indices (int64 tensor, each < 2^32) of stream (seed, stream)."""
    idx = index.to(torch.int64)
    idx = torch.where(idx >= (1 << 31), idx - (1 << 32), idx).to(torch.int32)
    return _u32_from_index(idx, _stream_key(seed, stream))


# ----------------------------------------------------------------------------
# inverse-CDF tables over every finite fp16 / bf16 value
# ----------------------------------------------------------------------------
def _finite_sorted(dtype: str) -> np.ndarray:
    if dtype == "fp16":
        pos_bits = np.arange(0, 0x7C00, dtype=np.uint16)
        pos = pos_bits.view(np.float16).astype(np.float64)
    elif dtype == "bf16":
        pos_bits = np.arange(0, 0x7F80, dtype=np.uint32) << 16
        pos = pos_bits.view(np.float32).astype(np.float64)
    else:
        raise ValueError(dtype)
    return np.concatenate([-pos[:0:-1], pos])  # -max .. -min, 0, min .. max


@functools.lru_cache(maxsize=16)
def _normal_table(dtype: str, sigma: float) -> tuple[np.ndarray, np.ndarray]:
    from scipy.special import ndtr

    vals = _finite_sorted(dtype)
    mids = (vals[:-1] + vals[1:]) * 0.5  # exact in float64
    cdf = ndtr(mids / sigma)
    thr = np.floor(cdf * 4294967296.0).astype(np.int64)
    thr = np.maximum.accumulate(thr)
    return thr, vals


@functools.lru_cache(maxsize=32)
def _normal_table_torch(dtype: str, sigma: float, device: str):
    thr, vals = _normal_table(dtype, sigma)
    tdt = torch.float16 if dtype == "fp16" else torch.bfloat16
    t_thr = torch.from_numpy(thr).to(device)
    t_val = torch.from_numpy(vals.astype(np.float32)).to(tdt).to(device)
    return t_thr, t_val


def _inverse_cdf(u: torch.Tensor, dtype: str, sigma: float) -> torch.Tensor:
    thr, vals = _normal_table_torch(dtype, float(sigma), str(u.device))
    idx = torch.searchsorted(thr, u, right=True)
    return vals[idx]


def normal_fp16(seed: int, stream: int, start: int, count: int, sigma: float,
                device="cpu") -> torch.Tensor:
    """fp16(N(0, sigma)) draws for elements [start, start+count) of one stream."""
    return _inverse_cdf(uniform_u32(seed, stream, start, count, device), "fp16", sigma)


def normal_bf16(seed: int, stream: int, start: int, count: int, sigma: float = 1.0,
                device="cpu") -> torch.Tensor:
    return _inverse_cdf(uniform_u32(seed, stream, start, count, device), "bf16", sigma)


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class Workload:
    cfg: int
    name: str
    E: int
    H: int
    F: int
    T: int
    k: int
    avg_bits: float
    sigma: float = 0.02
    outlier_frac: float = 0.0
    outlier_value: float = 0.2
    importance: str = "dirichlet"   # or "zipf"
    dirichlet_alpha: float = 1.0
    zipf_s: float = 1.1
    logits: str = "gaussian"         # or "zipf"

    @property
    def W_e(self) -> int:
        """Weight elements per expert: gate W1 [F x H], up W3 [F x H], down W2 [H x F]."""
        return 3 * self.H * self.F

    @property
    def sum_W(self) -> int:
        return self.E * self.W_e

    @property
    def budget_bits(self) -> int:
        return int(math.floor(self.avg_bits * self.sum_W))

    def seed(self, purpose: int) -> int:
        return 1000 * self.cfg + purpose


WORKLOADS = {
    1: Workload(1, "tiny-e8-h256-f512-t64-top2", E=8, H=256, F=512, T=64, k=2,
                avg_bits=4.5, importance="dirichlet", dirichlet_alpha=1.0),
    2: Workload(2, "mixtral-decode-e8-h4096-f14336-t16-top2", E=8, H=4096, F=14336, T=16,
                k=2, avg_bits=4.5, outlier_frac=0.001, outlier_value=0.2,
                importance="dirichlet", dirichlet_alpha=0.5),
    3: Workload(3, "finegrained-decode-e128-h2048-f768-t64-top8", E=128, H=2048, F=768,
                T=64, k=8, avg_bits=3.5, importance="zipf", logits="zipf"),
    4: Workload(4, "finegrained-prefill-e128-h2048-f768-t8192-top8", E=128, H=2048, F=768,
                T=8192, k=8, avg_bits=3.5, importance="zipf", logits="zipf"),
    5: Workload(5, "repage-e256-h7168-f2048-t128-top8", E=256, H=7168, F=2048, T=128, k=8,
                avg_bits=8.0, importance="dirichlet", dirichlet_alpha=1.0),
}

# Config 4 shares config 3's weights, bit allocation and routing distribution.
_WEIGHT_CFG = {1: 1, 2: 2, 3: 3, 4: 3, 5: 5}

# Dynamic repaging schedule: 20 steps, even = decode batch, odd = budget change.
REPAGE_AVG_BITS = [7.0, 6.0, 5.0, 4.0, 3.0, 3.75, 4.5, 5.25, 6.0, 6.0]


def schedule(wl: Workload) -> list[tuple[str, float | int]]:
    """[(kind, arg)]: ("decode", step_seed) or ("repage", avg_bits), 20 entries."""
    out = []
    for i in range(10):
        out.append(("decode", wl.seed(PURPOSE_SCHEDULE) * 100 + i))
        out.append(("repage", REPAGE_AVG_BITS[i]))
    return out


def budget_for(wl: Workload, avg_bits: float) -> int:
    return int(math.floor(avg_bits * wl.sum_W))


def weight_seed(wl: Workload) -> int:
    return 1000 * _WEIGHT_CFG[wl.cfg] + PURPOSE_WEIGHTS


def outlier_seed(wl: Workload) -> int:
    return 1000 * _WEIGHT_CFG[wl.cfg] + PURPOSE_OUTLIERS


def expert_weights(wl: Workload, e: int, start: int = 0, count: int | None = None,
                   device="cpu") -> torch.Tensor:
    """Flat fp16 master of expert e (W1 | W3 | W2, each row-major), elements [start, start+count)."""
    if count is None:
        count = wl.W_e - start
    w = normal_fp16(weight_seed(wl), e, start, count, wl.sigma, device)
    if wl.outlier_frac > 0.0:
        u = uniform_u32(outlier_seed(wl), e, start, count, device)
        thr = int(round(wl.outlier_frac * 4294967296.0))
        hit = u < thr
        # the sign comes from a bit of u that the threshold test does not decide
        sign_neg = ((u >> 3) & 1) == 1
        val = torch.tensor(wl.outlier_value, dtype=torch.float16, device=u.device)
        w = torch.where(hit, torch.where(sign_neg, -val, val), w)
    return w


def expert_weights_at(wl: Workload, e: int, index: torch.Tensor) -> torch.Tensor:
    """fp16 master of expert e at arbitrary flat element indices (same values as expert_weights)."""
    u = uniform_u32_at(weight_seed(wl), e, index)
    w = _inverse_cdf(u, "fp16", wl.sigma)
    if wl.outlier_frac > 0.0:
        uo = uniform_u32_at(outlier_seed(wl), e, index)
        thr = int(round(wl.outlier_frac * 4294967296.0))
        hit = uo < thr
        sign_neg = ((uo >> 3) & 1) == 1
        val = torch.tensor(wl.outlier_value, dtype=torch.float16, device=uo.device)
        w = torch.where(hit, torch.where(sign_neg, -val, val), w)
    return w


def expert_matrices(wl: Workload, e: int, device="cpu"):
    """(W1 [F,H], W3 [F,H], W2 [H,F]) fp16 views of one expert's master."""
    flat = expert_weights(wl, e, device=device)
    H, F = wl.H, wl.F
    w1 = flat[: F * H].view(F, H)
    w3 = flat[F * H: 2 * F * H].view(F, H)
    w2 = flat[2 * F * H:].view(H, F)
    return w1, w3, w2


def importance(wl: Workload) -> np.ndarray:
    """p_e (float64, sums to 1)."""
    rng = np.random.Generator(np.random.PCG64(1000 * _WEIGHT_CFG[wl.cfg] + PURPOSE_IMPORTANCE))
    if wl.importance == "dirichlet":
        return rng.dirichlet(np.full(wl.E, wl.dirichlet_alpha))
    if wl.importance == "zipf":
        return zipf_probs(wl)
    raise ValueError(wl.importance)


def zipf_probs(wl: Workload) -> np.ndarray:
    """pi_e with pi_rank ∝ rank^-s; a seeded permutation maps rank -> expert."""
    base = 1000 * _WEIGHT_CFG[wl.cfg] + PURPOSE_IMPORTANCE
    rng = np.random.Generator(np.random.PCG64(base))
    ranks = np.arange(1, wl.E + 1, dtype=np.float64)
    pr = ranks ** (-wl.zipf_s)
    pr /= pr.sum()
    expert_of_rank = rng.permutation(wl.E)
    pi = np.empty(wl.E)
    pi[expert_of_rank] = pr
    return pi


def router_logits(wl: Workload, T: int | None = None, seed: int | None = None) -> np.ndarray:
    T = wl.T if T is None else T
    s = wl.seed(PURPOSE_LOGITS) if seed is None else seed
    rng = np.random.Generator(np.random.PCG64(s))
    z = rng.standard_normal((T, wl.E))
    if wl.logits == "zipf":
        z = z + np.log(zipf_probs(wl))[None, :]
    return z


def topk_route(logits: np.ndarray, k: int) -> tuple[np.ndarray, np.ndarray]:
    """Top-k by logit (descending, ties to the lower expert id); weights = softmax
    over the k selected logits in float64, stored as float32."""
    T, E = logits.shape
    order = np.argsort(-logits, axis=1, kind="stable")[:, :k]
    sel = np.take_along_axis(logits, order, axis=1)
    mx = sel.max(axis=1, keepdims=True)
    ex = np.exp(sel - mx)
    w = ex / ex.sum(axis=1, keepdims=True)
    return order.astype(np.int32), w.astype(np.float32)


def routing(wl: Workload, T: int | None = None, seed: int | None = None):
    """(ids int32 [T,k], weights float32 [T,k]) for one batch."""
    return topk_route(router_logits(wl, T, seed), wl.k)


def activations(wl: Workload, T: int | None = None, seed: int | None = None,
                device="cpu") -> torch.Tensor:
    """bf16(N(0,1)) activations [T, H]."""
    T = wl.T if T is None else T
    s = wl.seed(PURPOSE_ACTIVATIONS) if seed is None else seed
    return normal_bf16(s, 0, 0, T * wl.H, 1.0, device).view(T, wl.H)


def scaled(wl: Workload, **changes) -> Workload:
    """A copy of a workload with some sizes changed (small parity cases)."""
    return dataclasses.replace(wl, **changes)


def fill_expert_weights(wl: Workload, e: int, out: torch.Tensor, chunk: int = 1 << 25) -> torch.Tensor:
    """Write expert e's full fp16 master into ``out`` (flat, W_e elements) in chunks,
    on ``out``'s device, bounding temporary memory."""
    assert out.numel() == wl.W_e and out.dtype == torch.float16
    flat = out.view(-1)
    for s in range(0, wl.W_e, chunk):
        n = min(chunk, wl.W_e - s)
        flat[s:s + n] = expert_weights(wl, e, s, n, device=out.device)
    return out
