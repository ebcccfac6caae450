"""Seeded synthetic inputs for the RG-LRU recurrent block.

This module only draws numbers: it holds none of the block's arithmetic, and it is the one
module that both the CUDA path (tests, bench) and the CPU oracle take inputs from, so both
sides see the same bytes.

Workloads follow the pages' description of the block and its initialisation ("Griffin
Guide: RecurrentGemma, RG-LRU & Hybrid Attention", section "1. Formulation of the RG-LRU
Gating Mechanism": ``a = sigma(Lambda)`` initialised so that ``a^c`` is uniform in
[0.9, 0.999], c = 8; the listing "PyTorch Implementation of RG-LRU and the Griffin Block",
``RGLRU._init_lambda``: draw u, take ``a = u^(1/c)`` and ``Lambda = logit(a)``).  The
shapes are RecurrentGemma-like synthetic workloads; no dataset or trained weight is used.

Recipe (all draws from one ``numpy.random.default_rng(seed)`` PCG64 stream, in this order):
  1. u ~ U[lo, hi] per channel (float64); Lambda = log(a / (1 - a)), a = u^(1/c) -> fp32
  2. W_a [H, dh, dh] ~ N(0, 1/dh)  (float32 draw, then rounded once to the act dtype)
  3. W_x [H, dh, dh] ~ N(0, 1/dh)
  4. conv_w [4, W] ~ N(0, 1/4) (variance 1/4) -> fp32;  conv_b = b_a = b_x = 0
  5. x [B, T, W] ~ N(0, 1), row b by row b, rounded once to the act dtype
  6. y [B, T, W] ~ N(0, 1), likewise
  7. (decode / state) h0 [B, W] ~ N(0, 1) fp32 and conv_tail0 [B, 3, W] ~ N(0, 1) in act dtype
  8. (packed) per row: document lengths ~ U{dmin..dmax} drawn until the row is full; the
     last document is cut at T; reset = 1 at every document start, t = 0 included.
bf16 values are stored as their 16 bits in numpy uint16 arrays (round to nearest even).
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

C_CONST = 8.0
CONV_WIDTH = 4


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seq_len: int
    heads: int
    head_dim: int
    dtype: str                   # "f32" or "bf16" (activations and gate weights)
    lam_lo: float = 0.9          # a^c ~ U[lam_lo, lam_hi]
    lam_hi: float = 0.999
    doc_len: Optional[tuple] = None   # (min, max) document length for packed rows
    decode_steps: int = 0        # > 0: a decode workload of this many single-token steps
    random_state: bool = False   # start from a random N(0,1) state instead of zero
    gelu_tanh: int = 0

    @property
    def width(self) -> int:
        return self.heads * self.head_dim

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads of the hot path, with their sizes.
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 256, 4, 64, "f32"),
    "rg2b_bf16": Workload("rg2b_bf16", 8, 2048, 10, 256, "bf16"),
    "long_bf16": Workload("long_bf16", 1, 65536, 16, 256, "bf16", lam_lo=0.99, lam_hi=0.9999),
    "decode_bf16": Workload("decode_bf16", 256, 1, 10, 256, "bf16", decode_steps=1024,
                            random_state=True),
    "packed_bf16": Workload("packed_bf16", 16, 8192, 24, 256, "bf16", doc_len=(64, 4096)),
}


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns the 16 stored bits."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bits to fp32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _to_act(a: np.ndarray, dtype: str) -> np.ndarray:
    return f32_to_bf16_bits(a) if dtype == "bf16" else np.ascontiguousarray(a, dtype=np.float32)


def make_params(wl: Workload, rng: np.random.Generator) -> dict:
    """Draws 1-4 of the recipe.  Gate weights are [H, dh_in, dh_out]."""
    W, H, dh = wl.width, wl.heads, wl.head_dim
    u = rng.uniform(wl.lam_lo, wl.lam_hi, size=W)
    a = u ** (1.0 / C_CONST)
    lam = np.log(a / (1.0 - a)).astype(np.float32)
    std = np.float32(1.0 / np.sqrt(dh))
    w_a = _to_act(rng.standard_normal((H, dh, dh), dtype=np.float32) * std, wl.dtype)
    w_x = _to_act(rng.standard_normal((H, dh, dh), dtype=np.float32) * std, wl.dtype)
    conv_w = (rng.standard_normal((CONV_WIDTH, W), dtype=np.float32) * np.float32(0.5))
    return dict(
        conv_w=np.ascontiguousarray(conv_w, dtype=np.float32),
        conv_b=np.zeros(W, np.float32),
        w_a=w_a, w_x=w_x,
        b_a=np.zeros(W, np.float32), b_x=np.zeros(W, np.float32),
        lam=lam,
    )


def make_activation(wl: Workload, rng: np.random.Generator, rows: int, seq: int) -> np.ndarray:
    """One [rows, seq, W] N(0,1) tensor in the act dtype, drawn row by row."""
    W = wl.width
    out = np.empty((rows, seq, W), dtype=np.uint16 if wl.dtype == "bf16" else np.float32)
    for b in range(rows):
        out[b] = _to_act(rng.standard_normal((seq, W), dtype=np.float32), wl.dtype)
    return out


def make_resets(wl: Workload, rng: np.random.Generator) -> Optional[np.ndarray]:
    """Draw 8: document-start mask [B, T] uint8, or None when the rows are unpacked."""
    if wl.doc_len is None:
        return None
    lo, hi = wl.doc_len
    reset = np.zeros((wl.batch, wl.seq_len), np.uint8)
    for b in range(wl.batch):
        t = 0
        while t < wl.seq_len:
            reset[b, t] = 1
            t += int(rng.integers(lo, hi + 1))
    return reset


def make_state(wl: Workload, rng: np.random.Generator):
    """Draw 7: (h0 [B, W] fp32, conv_tail0 [B, 3, W] act dtype)."""
    B, W = wl.batch, wl.width
    h0 = rng.standard_normal((B, W), dtype=np.float32)
    tail0 = _to_act(rng.standard_normal((B, CONV_WIDTH - 1, W), dtype=np.float32), wl.dtype)
    return h0, tail0


@dataclasses.dataclass
class Problem:
    wl: Workload
    params: dict
    x: np.ndarray
    y: np.ndarray
    reset: Optional[np.ndarray]
    h0: Optional[np.ndarray]
    tail0: Optional[np.ndarray]


def make_problem(wl: Workload, seed: int = 0) -> Problem:
    """A prefill problem: params, x, y [B, T, W], optional resets and initial state.

    For a decode workload (decode_steps > 0) x and y are [steps, B, W] (a fresh token per
    step) and the state is drawn after them.
    """
    rng = np.random.default_rng(seed)
    params = make_params(wl, rng)
    if wl.decode_steps > 0:
        x = make_activation(wl, rng, wl.decode_steps, wl.batch)
        y = make_activation(wl, rng, wl.decode_steps, wl.batch)
    else:
        x = make_activation(wl, rng, wl.batch, wl.seq_len)
        y = make_activation(wl, rng, wl.batch, wl.seq_len)
    h0 = tail0 = None
    if wl.random_state:
        h0, tail0 = make_state(wl, rng)
    reset = make_resets(wl, rng) if wl.decode_steps == 0 else None
    return Problem(wl, params, x, y, reset, h0, tail0)


def as_f32(a: np.ndarray) -> np.ndarray:
    """Exact fp32 view of an act-dtype array (bf16 bits are widened, fp32 passes through)."""
    return bf16_bits_to_f32(a) if a.dtype == np.uint16 else np.asarray(a, dtype=np.float32)
