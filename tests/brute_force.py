"""Brute-force reference for tiny inputs, written independently of the oracle.

Instead of walking slots, it builds the dense T x T mask over the per-token
partial slots by enumerating, for every query i and candidate key u, whether
the stride-aware causal mask lets i see the partial slot that ends at token u
("Multi-head Temporal Latent Attention", Method (2), Sec. 4.2, Fig. 2(c),
under the 0-based reading: every finished slot, plus the query's own slot
while it is being filled). Partial slots come from a pure-Python running sum
that restarts at every block start, the scores from an explicit per-head key
and value (no absorption), and the softmax from numpy over the masked row.
Pure-Python loops: only for T <= 16 or so.
"""
from __future__ import annotations

import math

import numpy as np


def dense_mask(T: int, s: int) -> np.ndarray:
    """mask[i, u] = True iff query i attends the partial slot that ends at token u."""
    m = np.zeros((T, T), dtype=bool)
    for i in range(T):
        for u in range(T):
            own = (u == i)
            finished = ((u + 1) % s == 0) and (u // s < i // s)
            m[i, u] = own or finished
    return m


def running_slots(x: np.ndarray, w: np.ndarray, s: int) -> np.ndarray:
    """P[t] = w[t] x[t] + (P[t-1] unless t starts a block); x [T,D], w [T]."""
    T, D = x.shape
    P = np.zeros((T, D))
    for t in range(T):
        prev = P[t - 1] if (t % s != 0) else np.zeros(D)
        P[t] = prev + w[t] * x[t]
    return P


def attention(q_full, P, w_uk, w_uv, s: int, d_c: int, scale: float) -> np.ndarray:
    """q_full [T,H,d_h+d_r] (already rotated), P [T,D] partial slots.
    Returns out [T,H,d_h] with explicit keys k = [W_UK P[:d_c]; P[d_c:]]."""
    T, H, _ = q_full.shape
    d_h = w_uk.shape[1]
    mask = dense_mask(T, s)
    out = np.zeros((T, H, d_h))
    for h in range(H):
        K = np.concatenate([P[:, :d_c] @ w_uk[h].T, P[:, d_c:]], axis=1)   # [T, d_h+d_r]
        V = P[:, :d_c] @ w_uv[h].T                                       # [T, d_h]
        scores = scale * (q_full[:, h, :] @ K.T)                         # [T, T]
        scores = np.where(mask, scores, -np.inf)
        scores = scores - scores.max(axis=1, keepdims=True)
        p = np.exp(scores)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ V
    return out


def softmax_scale(d_h: int, d_r: int) -> float:
    return 1.0 / math.sqrt(d_h + d_r)
