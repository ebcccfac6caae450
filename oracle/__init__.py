"""fp64 CPU oracle for the RG-LRU recurrent block -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the cpu_baseline / reference leg of
``bench.py`` may import this package.  The product (the CUDA library and its binding) never
imports, links or runs it, and it shares no code with the product: the arithmetic lives in
``rglru_oracle.c`` (plain C, fp64), and this file only marshals numpy arrays into it.

Inputs are the exact values handed to the GPU: fp32 arrays, or bf16 stored as their 16 bits
in uint16 arrays (widened exactly inside the C code).  Outputs and state are fp64.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rglru_oracle.c")
_LIB_PATH = os.path.join(_HERE, "librglru_oracle.so")
_lib = None

F32, BF16, F64 = 0, 1, 2
HIST = 3  # conv width 4 -> 3 past inputs


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (fp64, no fast-math, no FP contraction, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O3", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                               "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def load_library(path: str):
    """Open an oracle build at ``path`` and declare its entry points."""
    lib = ctypes.CDLL(path)
    P, I, D, L = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_long
    lib.rglru_oracle_gelu.restype = D
    lib.rglru_oracle_gelu.argtypes = [D, I]
    lib.rglru_oracle_prefill_unit.restype = I
    lib.rglru_oracle_prefill_unit.argtypes = [I, I, D, I, I, P, L, P, P, P, I, P, P, P,
                                              P, P, L, P, P, P, L, P, L, P]
    lib.rglru_oracle_prefill.restype = I
    lib.rglru_oracle_prefill.argtypes = [I, I, I, I, D, I, I, P, P, P, P, P, P, P,
                                         P, P, P, P, P, P, P, I, I]
    lib.rglru_oracle_backward.restype = I
    lib.rglru_oracle_backward.argtypes = [I, I, I, I, D, I, I] + [P] * 26
    lib.rglru_oracle_decode.restype = I
    lib.rglru_oracle_decode.argtypes = [I, I, I, D, I, I, P, P, P, P, P, P, P,
                                        P, P, P, P, P, P, I]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = load_library(build())
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _act(a: np.ndarray):
    if a.dtype == np.uint16:
        return np.ascontiguousarray(a), BF16
    return np.ascontiguousarray(a, dtype=np.float32), F32


def _f32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float32)


def gelu(v: float, tanh_form: int = 0) -> float:
    return _load().rglru_oracle_gelu(float(v), int(tanh_form))


def prefill(params: dict, x: np.ndarray, y: np.ndarray, heads: int,
            reset: Optional[np.ndarray] = None, h0: Optional[np.ndarray] = None,
            tail0: Optional[np.ndarray] = None, c: float = 8.0, gelu_tanh: int = 0,
            units: Optional[Sequence] = None, threads: int = 0):
    """Full-sequence prefill of x, y [B, T, W].

    Returns (out [B, T, W] fp64, h [B, W] fp64, tail [B, 3, W] fp64).  h0 / tail0 default to
    zero.  ``units`` = list of (b, head): only those sequences are computed (others stay 0).
    """
    lib = _load()
    x, dt = _act(x)
    y, dty = _act(y)
    assert dt == dty and x.shape == y.shape and x.ndim == 3
    B, T, W = x.shape
    dh = W // heads
    w_a, dtw = _act(params["w_a"])
    w_x, _ = _act(params["w_x"])
    assert dtw == dt, "gate weights are stored in the activation dtype"
    conv_w, conv_b = _f32(params["conv_w"]), _f32(params.get("conv_b"))
    b_a, b_x, lam = _f32(params.get("b_a")), _f32(params.get("b_x")), _f32(params["lam"])
    h = np.zeros((B, W)) if h0 is None else np.array(h0, dtype=np.float64, copy=True)
    tail = np.zeros((B, HIST, W)) if tail0 is None else tail_from_act(tail0).copy()
    out = np.zeros((B, T, W))
    rst = None if reset is None else np.ascontiguousarray(reset, dtype=np.uint8)
    uarr = None
    n_units = 0
    if units is not None:
        uarr = np.ascontiguousarray(np.array(units, dtype=np.int32).reshape(-1, 2))
        n_units = uarr.shape[0]
    rc = lib.rglru_oracle_prefill(B, T, heads, dh, c, gelu_tanh, dt, _p(conv_w), _p(conv_b),
                                  _p(w_a), _p(w_x), _p(b_a), _p(b_x), _p(lam), _p(x), _p(y),
                                  _p(rst), _p(h), _p(tail), _p(out), _p(uarr), n_units, threads)
    if rc != 0:
        raise RuntimeError("oracle prefill failed")
    return out, h, tail


def round_bf16(a: np.ndarray) -> np.ndarray:
    """fp64 -> the nearest bf16 value (ties to even), returned as fp64: 8 significant bits by
    frexp / rint, exact for the normal range (no detour through fp32, so no double rounding)."""
    a = np.asarray(a, dtype=np.float64)
    m, e = np.frexp(a)                       # a = m 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


def layer(params: dict, proj: dict, u: np.ndarray, heads: int, reset: Optional[np.ndarray] = None,
          h0: Optional[np.ndarray] = None, tail0: Optional[np.ndarray] = None, c: float = 8.0,
          gelu_tanh: int = 0, units: Optional[Sequence] = None, act_interface: bool = False):
    """The block with its projections ("Griffin Guide: RecurrentGemma, RG-LRU & Hybrid
    Attention", listing RecurrentBlock.forward: proj_in_1 / proj_in_2 before the branches,
    proj_out after the merge; RecurrentGemma's linear_x / linear_y / linear_out):

        x = u W_in_x,  y = u W_in_y,  z = block(x, y),  out = z W_out

    all in fp64 from the exact input values (u [B, T, D] and the weights w_in_x, w_in_y [D, W],
    w_out [W, D] of ``proj`` in the act dtype); the block is this oracle's prefill of x, y as
    fp64 inputs.  Returns (out [B, T, D], h [B, W], tail [B, 3, W], z [B, T, W]), fp64.
    ``units`` = list of (b, head) sequences to run (the others leave z at 0).

    act_interface: the three steps meet at the block's interface, whose activations are bf16
    tensors (the block takes x and y and returns z in the activation dtype): x, y and z are
    rounded to bf16 (nearest, ties to even) where they cross it, everything else stays fp64.
    The conv history the block keeps is then the bf16 x it was given."""
    lib = _load()
    u64 = as_f64(u)
    wx, wy, wo = as_f64(proj["w_in_x"]), as_f64(proj["w_in_y"]), as_f64(proj["w_out"])
    B, T, D = u64.shape
    W = wx.shape[1]
    dh = W // heads
    x = np.ascontiguousarray(np.matmul(u64, wx))
    y = np.ascontiguousarray(np.matmul(u64, wy))
    if act_interface:
        x, y = np.ascontiguousarray(round_bf16(x)), np.ascontiguousarray(round_bf16(y))
    w_a, dtw = _act(params["w_a"])
    w_x, _ = _act(params["w_x"])
    wes = 4 if dtw == F32 else 2
    conv_w = _f32(params["conv_w"])
    conv_b, b_a, b_x, lam = (_f32(params.get(k)) for k in ("conv_b", "b_a", "b_x", "lam"))
    h = np.zeros((B, W)) if h0 is None else np.array(h0, dtype=np.float64, copy=True)
    tail = np.zeros((B, HIST, W)) if tail0 is None else tail_from_act(tail0).copy()
    z = np.zeros((B, T, W))
    base = lambda arr, off, size: ctypes.c_void_p(arr.ctypes.data + off * size)  # noqa: E731
    todo = units if units is not None else [(b, hd) for b in range(B) for hd in range(heads)]
    for b, hd in todo:
        ch0 = hd * dh
        hb = np.ascontiguousarray(h[b, ch0:ch0 + dh])
        tb = np.ascontiguousarray(tail[b][:, ch0:ch0 + dh])
        zb = np.zeros((T, dh))
        rst = None if reset is None else np.ascontiguousarray(reset[b], dtype=np.uint8)
        rc = lib.rglru_oracle_prefill_unit(
            T, dh, c, gelu_tanh, F64, base(conv_w, ch0, 4), W,
            None if conv_b is None else base(conv_b, ch0, 4),
            base(w_a, hd * dh * dh, wes), base(w_x, hd * dh * dh, wes), dtw,
            None if b_a is None else base(b_a, ch0, 4), None if b_x is None else base(b_x, ch0, 4),
            base(lam, ch0, 4), base(x, b * T * W + ch0, 8), base(y, b * T * W + ch0, 8), W,
            _p(rst), _p(hb), _p(tb), dh, _p(zb), dh, None)
        if rc != 0:
            raise RuntimeError("oracle layer: prefill_unit failed")
        z[b, :, ch0:ch0 + dh] = zb
        h[b, ch0:ch0 + dh] = hb
        tail[b][:, ch0:ch0 + dh] = tb
    out = np.matmul(round_bf16(z) if act_interface else z, wo)
    return out, h, tail, z


def as_f64(a: np.ndarray) -> np.ndarray:
    """Exact fp64 copy of an act-dtype array (bf16 bits widened)."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return np.ascontiguousarray((a.astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    return np.ascontiguousarray(a, dtype=np.float64)


def prefill_unit_decay(params: dict, x: np.ndarray, y: np.ndarray, heads: int, b: int, head: int,
                       reset: Optional[np.ndarray] = None, c: float = 8.0):
    """One (b, head) sequence from zero state; returns (out [T, dh], a_t [T, dh])."""
    lib = _load()
    x, dt = _act(x)
    y, _ = _act(y)
    B, T, W = x.shape
    dh = W // heads
    w_a, _ = _act(params["w_a"])
    w_x, _ = _act(params["w_x"])
    es = 4 if dt == F32 else 2
    ch0 = head * dh
    conv_w = _f32(params["conv_w"])
    conv_b, b_a, b_x, lam = (_f32(params.get(k)) for k in ("conv_b", "b_a", "b_x", "lam"))
    h = np.zeros(dh)
    tail = np.zeros((HIST, dh))
    out = np.zeros((T, dh))
    a_out = np.zeros((T, dh))
    base = lambda arr, off, size: ctypes.c_void_p(arr.ctypes.data + off * size)  # noqa: E731
    rst = None if reset is None else np.ascontiguousarray(reset[b], dtype=np.uint8)
    rc = lib.rglru_oracle_prefill_unit(
        T, dh, c, 0, dt, base(conv_w, ch0, 4), W,
        None if conv_b is None else base(conv_b, ch0, 4),
        base(w_a, head * dh * dh, es), base(w_x, head * dh * dh, es), dt,
        None if b_a is None else base(b_a, ch0, 4), None if b_x is None else base(b_x, ch0, 4),
        base(lam, ch0, 4), base(x, b * T * W + ch0, es), base(y, b * T * W + ch0, es), W,
        _p(rst), _p(h), _p(tail), dh, _p(out), dh, _p(a_out))
    if rc != 0:
        raise RuntimeError("oracle prefill_unit failed")
    return out, a_out


def decode(params: dict, x: np.ndarray, y: np.ndarray, heads: int, h: np.ndarray,
           tail: np.ndarray, reset: Optional[np.ndarray] = None, c: float = 8.0,
           gelu_tanh: int = 0, threads: int = 0):
    """One decode step for x, y [B, W]; h [B, W] and tail [B, 3, W] (fp64) are updated in
    place.  Returns out [B, W] fp64."""
    lib = _load()
    x, dt = _act(x)
    y, _ = _act(y)
    B, W = x.shape
    dh = W // heads
    w_a, _ = _act(params["w_a"])
    w_x, _ = _act(params["w_x"])
    assert h.dtype == np.float64 and h.flags.c_contiguous
    assert tail.dtype == np.float64 and tail.flags.c_contiguous
    conv_w, conv_b = _f32(params["conv_w"]), _f32(params.get("conv_b"))
    b_a, b_x, lam = _f32(params.get("b_a")), _f32(params.get("b_x")), _f32(params["lam"])
    rst = None if reset is None else np.ascontiguousarray(reset, dtype=np.uint8)
    out = np.zeros((B, W))
    rc = lib.rglru_oracle_decode(B, heads, dh, c, gelu_tanh, dt, _p(conv_w), _p(conv_b),
                                 _p(w_a), _p(w_x), _p(b_a), _p(b_x), _p(lam), _p(x), _p(y),
                                 _p(rst), _p(h), _p(tail), _p(out), threads)
    if rc != 0:
        raise RuntimeError("oracle decode failed")
    return out


def tail_from_act(tail0: np.ndarray) -> np.ndarray:
    """fp64 copy of an act-dtype conv history (bf16 bits or fp32)."""
    if tail0.dtype == np.uint16:
        return np.ascontiguousarray((tail0.astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    return np.ascontiguousarray(tail0, dtype=np.float64)


def prefill_units(params: dict, x: np.ndarray, y: np.ndarray, heads: int, units: Sequence,
                  reset: Optional[np.ndarray] = None, h0: Optional[np.ndarray] = None,
                  tail0: Optional[np.ndarray] = None, c: float = 8.0, gelu_tanh: int = 0,
                  workers: int = 0):
    """Prefill of selected (b, head) sequences only, without materialising [B, T, W] outputs.

    Returns {(b, head): (out [T, dh], h [dh], tail [3, dh])}, fp64.  Sequences run in parallel
    threads (the C call releases the GIL); each one is the plain sequential definition.
    """
    from concurrent.futures import ThreadPoolExecutor
    lib = _load()
    B, T, W = x.shape
    dh = W // heads
    _, dt = _act(x[:1, :1])
    es = 4 if dt == F32 else 2
    w_a, _ = _act(params["w_a"])
    w_x, _ = _act(params["w_x"])
    conv_w = _f32(params["conv_w"])
    conv_b, b_a, b_x, lam = (_f32(params.get(k)) for k in ("conv_b", "b_a", "b_x", "lam"))
    base = lambda arr, off, size: ctypes.c_void_p(arr.ctypes.data + off * size)  # noqa: E731

    def one(unit):
        b, hd = unit
        ch0 = hd * dh
        xs, _ = _act(x[b, :, ch0:ch0 + dh])
        ys, _ = _act(y[b, :, ch0:ch0 + dh])
        h = np.zeros(dh) if h0 is None else np.array(h0[b, ch0:ch0 + dh], dtype=np.float64)
        tail = (np.zeros((HIST, dh)) if tail0 is None
                else np.ascontiguousarray(tail_from_act(tail0[b][:, ch0:ch0 + dh])))
        out = np.zeros((T, dh))
        rst = None if reset is None else np.ascontiguousarray(reset[b], dtype=np.uint8)
        rc = lib.rglru_oracle_prefill_unit(
            T, dh, c, gelu_tanh, dt, base(conv_w, ch0, 4), W,
            None if conv_b is None else base(conv_b, ch0, 4),
            base(w_a, hd * dh * dh, es), base(w_x, hd * dh * dh, es), dt,
            None if b_a is None else base(b_a, ch0, 4), None if b_x is None else base(b_x, ch0, 4),
            base(lam, ch0, 4), _p(xs), _p(ys), dh, _p(rst), _p(h), _p(tail), dh, _p(out), dh, None)
        if rc != 0:
            raise RuntimeError("oracle prefill_unit failed")
        return (b, hd), (out, h, tail)

    n = workers or min(len(units), max(1, os.cpu_count() or 1))
    with ThreadPoolExecutor(max_workers=n) as ex:
        return dict(ex.map(one, [tuple(u) for u in units]))


def backward(params: dict, x: np.ndarray, y: np.ndarray, heads: int, dout: np.ndarray,
             reset: Optional[np.ndarray] = None, h0: Optional[np.ndarray] = None,
             tail0: Optional[np.ndarray] = None, dh_final: Optional[np.ndarray] = None,
             dtail_final: Optional[np.ndarray] = None, c: float = 8.0, gelu_tanh: int = 0) -> dict:
    """Exact fp64 gradients of L = <dout, out> + <dh_final, h_T> + <dtail_final, tail_T> for the
    prefill of x, y [B, T, W] from the state (h0, tail0) (zero when None).

    Returns a dict of fp64 arrays: dx, dy [B, T, W]; dh0 [B, W]; dtail0 [B, 3, W];
    dconv_w [4, W]; dconv_b, db_a, db_x, dlam [W]; dw_a, dw_x [H, dh, dh].
    """
    lib = _load()
    x, dt = _act(x)
    y, _ = _act(y)
    dout, dtd = _act(dout)
    assert dtd == dt and dout.shape == x.shape
    B, T, W = x.shape
    dh = W // heads
    w_a, _ = _act(params["w_a"])
    w_x, _ = _act(params["w_x"])
    conv_w, conv_b = _f32(params["conv_w"]), _f32(params.get("conv_b"))
    b_a, b_x, lam = _f32(params.get("b_a")), _f32(params.get("b_x")), _f32(params["lam"])
    f64 = lambda a: None if a is None else np.ascontiguousarray(a, dtype=np.float64)  # noqa: E731
    h0 = f64(h0)
    tail0 = None if tail0 is None else tail_from_act(tail0)
    dh_final, dtail_final = f64(dh_final), f64(dtail_final)
    rst = None if reset is None else np.ascontiguousarray(reset, dtype=np.uint8)
    g = {"dx": np.zeros((B, T, W)), "dy": np.zeros((B, T, W)), "dh0": np.zeros((B, W)),
         "dtail0": np.zeros((B, HIST, W)), "dconv_w": np.zeros((4, W)), "dconv_b": np.zeros(W),
         "dw_a": np.zeros((heads, dh, dh)), "dw_x": np.zeros((heads, dh, dh)),
         "db_a": np.zeros(W), "db_x": np.zeros(W), "dlam": np.zeros(W)}
    rc = lib.rglru_oracle_backward(
        B, T, heads, dh, c, gelu_tanh, dt, _p(conv_w), _p(conv_b), _p(w_a), _p(w_x), _p(b_a),
        _p(b_x), _p(lam), _p(x), _p(y), _p(rst), _p(h0), _p(tail0), _p(dout), _p(dh_final),
        _p(dtail_final), _p(g["dx"]), _p(g["dy"]), _p(g["dh0"]), _p(g["dtail0"]),
        _p(g["dconv_w"]), _p(g["dconv_b"]), _p(g["dw_a"]), _p(g["dw_x"]), _p(g["db_a"]),
        _p(g["db_x"]), _p(g["dlam"]))
    if rc != 0:
        raise RuntimeError("oracle backward failed")
    return g

