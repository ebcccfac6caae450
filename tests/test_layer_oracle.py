"""Pins of the layer oracle (the block with its projections, oracle.layer).

The projections are plain fp64 matmuls around the block oracle, so they are pinned by
structure rather than by retyping them: with projection matrices that pick one input channel
per output channel (a permutation, scaled by powers of two so that every product is exact),
x, y and out are fixed by indexing alone, and the layer must equal the block oracle run on the
indexed inputs.  A permutation that is not its own inverse makes a transposed weight visible;
a planted transposition is caught.
"""

import os

import numpy as np
import torch
import pytest

import oracle
from gated_linear_recurrence_conv1d_b200 import inputs


def _selector(rows, cols, pick, scale):
    """[rows, cols] matrix with M[pick[j], j] = scale[j] (bf16-exact powers of two)."""
    m = np.zeros((rows, cols), np.float32)
    m[pick, np.arange(cols)] = scale
    return m


def _bf16(a):
    return inputs.f32_to_bf16_bits(a)


def _case(D, heads=2, dh=16, T=24, seed=0):
    W = heads * dh
    wl = inputs.WORKLOADS["packed_bf16"].scaled(batch=2, seq_len=T, heads=heads, head_dim=dh, doc_len=(5, 12))
    prob = inputs.make_problem(wl, seed=seed)
    rng = np.random.default_rng(seed + 1)
    u = _bf16(rng.standard_normal((2, T, D)).astype(np.float32))
    px = rng.permutation(D)[:W]                       # x_j = sx_j u_{px_j}
    py = rng.permutation(D)[:W]
    po = rng.permutation(max(D, W))[:D] % W           # out_d = so_d z_{po_d}
    sx = 2.0 ** rng.integers(-2, 3, W)
    sy = 2.0 ** rng.integers(-2, 3, W)
    so = 2.0 ** rng.integers(-2, 3, D)
    proj = {"w_in_x": _bf16(_selector(D, W, px, sx)), "w_in_y": _bf16(_selector(D, W, py, sy)),
            "w_out": _bf16(_selector(W, D, po, so))}
    return prob, u, proj, (px, py, po, sx, sy, so)


def _check_layer(layer_fn, D):
    prob, u, proj, (px, py, po, sx, sy, so) = _case(D)
    heads = prob.wl.heads
    uf = inputs.as_f32(u)
    x_ref = _bf16((uf[:, :, px] * sx).astype(np.float32))  # exact: bf16 times a power of two
    y_ref = _bf16((uf[:, :, py] * sy).astype(np.float32))
    z_ref, h_ref, t_ref = oracle.prefill(prob.params, x_ref, y_ref, heads, reset=prob.reset)
    out_ref = z_ref[:, :, po] * so
    out, h, tail, z = layer_fn(prob.params, proj, u, heads, reset=prob.reset)
    np.testing.assert_array_equal(z, z_ref)
    np.testing.assert_array_equal(out, out_ref)
    np.testing.assert_array_equal(h, h_ref)
    np.testing.assert_array_equal(tail, t_ref)


@pytest.mark.parametrize("D", [32, 48])
def test_layer_projections_by_channel_selection(D):
    _check_layer(oracle.layer, D)


def test_layer_with_identity_projections_is_the_block():
    wl = inputs.WORKLOADS["rg2b_bf16"].scaled(batch=1, seq_len=30, heads=2, head_dim=16, random_state=True)
    prob = inputs.make_problem(wl, seed=5)
    eye = _bf16(np.eye(32, dtype=np.float32))
    proj = {"w_in_x": eye, "w_in_y": eye, "w_out": eye}
    out, h, tail, _ = oracle.layer(prob.params, proj, prob.x, 2, h0=prob.h0, tail0=prob.tail0)
    ref, rh, rt = oracle.prefill(prob.params, prob.x, prob.x, 2, h0=prob.h0, tail0=prob.tail0)
    np.testing.assert_array_equal(out, ref)
    np.testing.assert_array_equal(h, rh)


def test_transposed_projection_is_caught():
    """A planted mistake: the input projection applied transposed (W^T instead of W, both
    D x D).  The selection pin must fail on it."""
    src = open(os.path.join(os.path.dirname(oracle.__file__), "__init__.py")).read()
    old = "x = np.ascontiguousarray(np.matmul(u64, wx))"
    assert src.count(old) == 1
    ns = {"__name__": "oracle_mutant", "__file__": oracle.__file__}
    exec(compile(src.replace(old, "x = np.ascontiguousarray(np.matmul(u64, wx.T))"), "oracle_mutant", "exec"), ns)
    ns["_lib"] = oracle._load()
    with pytest.raises(AssertionError):
        _check_layer(ns["layer"], 32)


def test_round_bf16_is_nearest_even_bf16():
    """The layer oracle's interface rounding: torch's fp32 -> bf16 conversion (round to nearest
    even) on fp32-representable values over 12 decades, and the ties at 1 + 2^-8 (to 1) and
    1 + 3 2^-8 (to 1 + 2^-6)."""
    rng = np.random.default_rng(0)
    a = (rng.standard_normal(100000) * 10.0 ** rng.uniform(-6, 6, 100000)).astype(np.float32)
    want = torch.from_numpy(a).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(oracle.round_bf16(a.astype(np.float64)), want)
    ties = oracle.round_bf16(np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8)]))
    np.testing.assert_array_equal(ties, [1.0, 1 + 2.0 ** -6, -1.0])
