"""Dynamic error compensation of salient input channels, float64.

DecDEC summary (blog summary of "DecDEC: A Systems Approach to Advancing
Low-Bit LLM Quantization"), 3.1: each linear W^ x of the quantized model
becomes (W^ + R (.) M) x, where R = W - W^ is the residual between the
full-precision and the quantized weights and M is a binary mask that keeps a
small, structured part of R. 3.2: M selects whole input channels, those whose
activations have the largest magnitudes (salient channels: an outlier
activation multiplies the small quantization error of its weight column);
Figure 4: replacing the channels of W^ by their FP16 values in descending
order of |x| lowers the error of W^ x against W x much faster than in random
order.

Readings taken where the pages leave the step open:
* M is chosen per input row: per token for the gate and up projections
  (they share x, so they share the mask), per routed position for the down
  projection (its input is that position's h). A row keeps its n channels of
  largest |x_c|, ties to the lower channel index; all channels when n is at
  least the row length.
* R is taken against the fp16 master W and the expert's current W^ = s k, so
  on a kept channel the compensated weights are exactly the fp16 master values
  (Figure 4's "replaced with FP16 counterparts").
* The SwiGLU expert FFN (see ffn.py) compensates all three projections; h is
  formed from the compensated g and v, and the down projection's mask is taken
  on that h.
"""
from __future__ import annotations

from typing import Callable

import numpy as np

from .ffn import silu


def salient_channels(row, n: int) -> np.ndarray:
    """Indices (ascending) of the n entries of largest |row|, ties to the
    lower index; every index when n >= len(row)."""
    row = np.asarray(row, dtype=np.float64)
    L = row.shape[0]
    if n >= L:
        return np.arange(L)
    if n <= 0:
        return np.zeros(0, dtype=np.int64)
    # primary key |x| descending, secondary the index ascending
    order = np.lexsort((np.arange(L), -np.abs(row)))
    return np.sort(order[:n])


def compensated_linear(w_hat: np.ndarray, w: np.ndarray, x: np.ndarray, n: int) -> np.ndarray:
    """(W^ + R (.) M) x for one input row x, M keeping x's n salient channels."""
    sel = salient_channels(x, n)
    return w_hat @ x + (w[:, sel] - w_hat[:, sel]) @ x[sel]


def expert_ffn_compensated(x_rows, hat, master, n: int, down_masks=None) -> np.ndarray:
    """y [rows, H] for input rows x [rows, H]; hat = (W1^, W3^, W2^), master =
    (W1, W3, W2) in float64 (the fp16 values). down_masks: optional kept
    channels of each row's h (a list of index arrays) to use instead of
    choosing them here -- several choices are correct where |h| values tie or
    nearly tie at the cut, so a parity check takes the device's choice, after
    checking it is one of them."""
    w1h, w3h, w2h = hat
    w1, w3, w2 = master
    out = []
    for r, x in enumerate(np.asarray(x_rows, dtype=np.float64)):
        g = compensated_linear(w1h, w1, x, n)
        v = compensated_linear(w3h, w3, x, n)
        h = silu(g) * v
        if down_masks is None:
            out.append(compensated_linear(w2h, w2, h, n))
        else:
            sel = np.asarray(down_masks[r])
            out.append(w2h @ h + (w2[:, sel] - w2h[:, sel]) @ h[sel])
    return np.stack(out) if out else np.zeros((0, w2h.shape[0]))


def moe_ffn_compensated(x, ids, w, expert_weights: Callable, expert_masters: Callable, E: int,
                        n: int, tokens=None, down_masks=None) -> np.ndarray:
    """The routed layer of ffn.moe_ffn with every projection compensated.
    expert_weights(e) -> (W1^, W3^, W2^); expert_masters(e) -> (W1, W3, W2);
    down_masks: optional {(t, j): kept channels of that slot's h}."""
    x = np.asarray(x, dtype=np.float64)
    ids = np.asarray(ids)
    w = np.asarray(w, dtype=np.float64)
    T, H = x.shape
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    out = np.zeros((len(tokens), H), dtype=np.float64)
    for e in range(E):
        rows = [(oi, t, j) for oi, t in enumerate(tokens) for j in range(ids.shape[1])
                if ids[t, j] == e]
        if not rows:
            continue
        masks = None if down_masks is None else [down_masks[(t, j)] for _, t, j in rows]
        y = expert_ffn_compensated(np.stack([x[t] for _, t, _ in rows]), expert_weights(e),
                                   expert_masters(e), n, masks)
        for r, (oi, t, j) in enumerate(rows):
            out[oi] += w[t, j] * y[r]
    return out


def is_valid_choice(row, kept, n: int, tol: float, rel: float = 0.0) -> bool:
    """True when `kept` (n distinct indices, or every index when n >= len(row))
    is a largest-|row| choice up to rounding: no left-out entry a exceeds a
    kept one c by more than tol + rel * (|a| + |c|). For checking a choice made
    on rounded values: if each compared value may be off by a relative rel
    (its rounding) plus tol / 2 (the error before it), two values whose
    rounded forms are ordered one way may truly differ the other way by at
    most that much. The extreme pair (largest left out, smallest kept) decides
    it, since the bound grows with both values."""
    row = np.abs(np.asarray(row, dtype=np.float64))
    L = row.shape[0]
    kept = np.asarray(kept)
    if n >= L:
        return np.array_equal(np.sort(kept), np.arange(L))
    if len(kept) != n or len(set(kept.tolist())) != n:
        return False
    rest = np.setdiff1d(np.arange(L), kept)
    a, c = row[rest].max(), row[kept].min()
    return a - c <= tol + rel * (a + c)


def error_curve(w_hat: np.ndarray, w: np.ndarray, x: np.ndarray, order) -> np.ndarray:
    """Figure 4's measurement for one row x: the mean squared error between
    W x and the output after the first i channels of `order` are replaced by
    their fp16 values, for i = 0 .. len(order)."""
    x = np.asarray(x, dtype=np.float64)
    ref = w @ x
    cur = w_hat @ x
    r = w - w_hat
    errs = [np.mean((cur - ref) ** 2)]
    for c in order:
        cur = cur + r[:, c] * x[c]
        errs.append(np.mean((cur - ref) ** 2))
    return np.asarray(errs)
