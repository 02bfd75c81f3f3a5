"""Dequantize-then-multiply routed expert FFN, float64 throughout.

PagedWeight, "Dynamic Paging": the pass fetches the needed experts' pages and
dequantizes them on the fly; DecDEC summary, 2.2: weight-only quantization
loads quantized weights, dequantizes them, and multiplies with
full-precision activations. The FFN form is SwiGLU (reading taken: the pages
do not name it): for token x and expert e with dequantized weights
W1^ = s k1 (gate), W3^ = s k3 (up), W2^ = s k2 (down),

    g = W1^ x,  v = W3^ x,  h = g / (1 + exp(-g)) * v,  y = W2^ h,

and the layer output is out[t] = sum_j w[t, j] * y_{t, j} over the token's
top-k slots j (ids outside [0, E) contribute nothing).

Every product and sum is float64 with no intermediate rounding; the CUDA path
rounds h and out to bf16, which the parity tolerance covers.
"""
from __future__ import annotations

from typing import Callable

import numpy as np


def silu(g: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g))


def gate_up(x: np.ndarray, w1: np.ndarray, w3: np.ndarray):
    """(g, v) for rows x [n, H] and dequantized W1, W3 [F, H]."""
    return x @ w1.T, x @ w3.T


def expert_ffn(x: np.ndarray, w1: np.ndarray, w3: np.ndarray, w2: np.ndarray) -> np.ndarray:
    """y [n, H] for rows x [n, H]."""
    g, v = gate_up(x, w1, w3)
    h = silu(g) * v
    return h @ w2.T


def moe_ffn(x: np.ndarray, ids: np.ndarray, w: np.ndarray,
            expert_weights: Callable[[int], tuple[np.ndarray, np.ndarray, np.ndarray]],
            E: int, tokens=None) -> np.ndarray:
    """out [len(tokens), H] in float64.

    x: [T, H] activations (float64 values of the bf16 inputs); ids [T, k];
    w: [T, k] top-k weights; expert_weights(e) -> dequantized (W1^, W3^, W2^).
    tokens: optional subset of token indices to evaluate (default: all).
    """
    x = np.asarray(x, dtype=np.float64)
    ids = np.asarray(ids)
    w = np.asarray(w, dtype=np.float64)
    T, H = x.shape
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    out = np.zeros((len(tokens), H), dtype=np.float64)
    for e in range(E):
        rows = []
        for oi, t in enumerate(tokens):
            for j in range(ids.shape[1]):
                if ids[t, j] == e:
                    rows.append((oi, t, j))
        if not rows:
            continue
        w1, w3, w2 = expert_weights(e)
        xs = np.stack([x[t] for _, t, _ in rows])
        y = expert_ffn(xs, w1, w3, w2)
        for r, (oi, t, j) in enumerate(rows):
            out[oi] += w[t, j] * y[r]
    return out
