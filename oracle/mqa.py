"""fp64 oracle of Griffin's local sliding-window multi-query attention -- TEST INFRASTRUCTURE.

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference leg may use this
module; the CUDA library never imports or runs it.

What it computes ("Griffin Guide: RecurrentGemma, RG-LRU & Hybrid Attention", "2. Local
Sliding-Window Multi-Query Attention (MQA)" and "3. Bounding the Key-Value Cache Footprint";
the "Griffin" notes, "Local Attention Path"):

  * H query heads share one key head and one value head (H_KV = 1);
  * token t attends to the window N(t) = {i : t - w < i <= t} of earlier positions, itself
    included:  y_t = sum_{i in N(t)} softmax_i(s q_t . k_i) v_i;
  * rotary position embeddings are applied to queries and keys;
  * a decode step keeps only the last w keys and values, in a ring buffer indexed by
    position mod w.

Readings where the pages are silent: the score scale s is a parameter (1/sqrt(head_dim) by
default, the usual scaled dot product; the pages write softmax(q . k) without one); RoPE rotates
the pairs (j, j + d/2) of a head of width d by the angle p * base^(-2j/d) at position p, base
10000 (the "rotate half" arrangement).  Inputs are the exact values given to the GPU (bf16 bits
widened); everything else is fp64, in the order of the definition.
"""

from __future__ import annotations

from typing import Optional

import numpy as np


def _f64(a: np.ndarray) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def rope(x: np.ndarray, pos: np.ndarray, base: float = 10000.0) -> np.ndarray:
    """Rotary embedding of x [..., d] at integer positions pos (broadcast over the leading
    axes): the pairs (j, j + d/2) turn by pos * base^(-2j/d)."""
    x = _f64(x)
    d = x.shape[-1]
    half = d // 2
    inv = base ** (-2.0 * np.arange(half) / d)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * inv
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def prefill(q: np.ndarray, k: np.ndarray, v: np.ndarray, window: int, pos0: int = 0,
            scale: Optional[float] = None, base: float = 10000.0) -> np.ndarray:
    """q [B, T, H, d], k, v [B, T, d] (one key / value head) at positions pos0 .. pos0+T-1.
    Returns y [B, T, H, d] fp64."""
    qf, kf, vf = _f64(q), _f64(k), _f64(v)
    B, T, H, d = qf.shape
    s = (1.0 / np.sqrt(d)) if scale is None else scale
    pos = pos0 + np.arange(T)
    qr = rope(qf, pos[None, :, None], base)          # [B, T, H, d]
    kr = rope(kf, pos[None, :], base)                # [B, T, d]
    y = np.zeros((B, T, H, d))
    for b in range(B):
        for t in range(T):
            lo = max(0, t - window + 1)
            keys = kr[b, lo:t + 1]                   # the window N(t), oldest first
            vals = vf[b, lo:t + 1]
            for h in range(H):
                sc = s * (keys @ qr[b, t, h])
                e = np.exp(sc - sc.max())
                y[b, t, h] = (e / e.sum()) @ vals
    return y


class RingCache:
    """The decode-time key / value store of one batch row: w slots, position p in slot p mod w;
    keys are kept after their rotation, values as given."""

    def __init__(self, window: int, d: int):
        self.w = window
        self.k = np.zeros((window, d))
        self.v = np.zeros((window, d))
        self.filled = 0          # positions seen so far

    def push(self, k_rot: np.ndarray, v: np.ndarray, pos: int):
        self.k[pos % self.w] = k_rot
        self.v[pos % self.w] = v
        self.filled = pos + 1

    def window_of(self, pos: int):
        lo = max(0, pos - self.w + 1)
        idx = [p % self.w for p in range(lo, pos + 1)]
        return self.k[idx], self.v[idx]


def decode_step(cache: RingCache, q: np.ndarray, k: np.ndarray, v: np.ndarray, pos: int,
                scale: Optional[float] = None, base: float = 10000.0) -> np.ndarray:
    """One token of one row: q [H, d], k, v [d] at position pos; the cache is updated first
    (the token attends to itself).  Returns y [H, d]."""
    qf, kf, vf = _f64(q), _f64(k), _f64(v)
    H, d = qf.shape
    s = (1.0 / np.sqrt(d)) if scale is None else scale
    cache.push(rope(kf, np.array(pos), base), vf, pos)
    keys, vals = cache.window_of(pos)
    qr = rope(qf, np.array(pos), base)
    y = np.zeros((H, d))
    for h in range(H):
        sc = s * (keys @ qr[h])
        e = np.exp(sc - sc.max())
        y[h] = (e / e.sum()) @ vals
    return y
