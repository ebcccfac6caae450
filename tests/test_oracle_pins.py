"""Pins of the fp64 CPU oracle against what the pages and the mathematics fix.

None of these checks re-types the oracle's loop: each one uses another formulation
(closed form, unrolled double sum, dense block-diagonal matrix, torch conv1d, the power form
a^(c r) instead of the log form, sqrt(1 - a^2) instead of sqrt(-expm1(2 log a)), scipy's
normal CDF for GeLU) or an invariant the pages state, so that a dropped term, a wrong sign or
index, or a transposed operand in the oracle fails at least one of them.

Sources ("Griffin Guide: RecurrentGemma, RG-LRU & Hybrid Attention"):
  gates / decay / update ......... "1. Formulation of the RG-LRU Gating Mechanism"
  unit variance .................. "2. The Role of Square-Root Variance Normalization"
  r -> 0 freezes h ............... "3. Super-Exponential Context Preservation"
  conv k = 4, GeLU merge ......... "1. Temporal Filtering via Separable 1D Convolutions",
                                   "2. Non-Linear Multiplicative Gating with GeLU"
  block-diagonal gates ........... "3. Block-Diagonal Sharding for Zero-Communication ..."
  conv padding / carry / F.gelu .. "1. PyTorch Implementation of RG-LRU and the Griffin Block"
"""

import json
import math
import os

import numpy as np
import pytest
import scipy.linalg
import scipy.special
import torch

import oracle
from gated_linear_recurrence_conv1d_b200 import inputs

C = 8.0
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _params(W, H, dh, rng, dtype="f32", bias=True, lam_range=(0.9, 0.999)):
    u = rng.uniform(*lam_range, size=W)
    a = u ** (1 / C)
    lam = np.log(a / (1 - a)).astype(np.float32)
    p = dict(
        conv_w=rng.standard_normal((4, W)).astype(np.float32) * 0.5,
        conv_b=(rng.standard_normal(W).astype(np.float32) * 0.3) if bias else np.zeros(W, np.float32),
        w_a=(rng.standard_normal((H, dh, dh)) / math.sqrt(dh)).astype(np.float32),
        w_x=(rng.standard_normal((H, dh, dh)) / math.sqrt(dh)).astype(np.float32),
        b_a=(rng.standard_normal(W).astype(np.float32) * 0.5) if bias else np.zeros(W, np.float32),
        b_x=(rng.standard_normal(W).astype(np.float32) * 0.5) if bias else np.zeros(W, np.float32),
        lam=lam,
    )
    if dtype == "bf16":
        p["w_a"] = inputs.f32_to_bf16_bits(p["w_a"])
        p["w_x"] = inputs.f32_to_bf16_bits(p["w_x"])
    return p


def _gelu_ref(v):
    """GeLU(v) = v * Phi(v) with scipy's normal CDF (an independent library routine)."""
    v = np.asarray(v, dtype=np.float64)
    return v * scipy.special.ndtr(v)


# ---------------------------------------------------------------- GeLU -------------------

def test_gelu_spot_values():
    assert oracle.gelu(0.0) == 0.0
    assert oracle.gelu(8.0) == pytest.approx(8.0, rel=1e-15)
    assert oracle.gelu(-8.0) == pytest.approx(-8.0 * scipy.special.ndtr(-8.0), rel=1e-12)
    for v in np.linspace(-6, 6, 97):
        assert oracle.gelu(v) == pytest.approx(_gelu_ref(v), rel=1e-13, abs=1e-300)


def test_gelu_tanh_form_matches_torch():
    """The tanh variant against an independent implementation of the same formula: torch's
    fp64 gelu(approximate="tanh") at 121 points across [-8, 8] (both sides evaluate
    0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))), so they agree to rounding)."""
    import torch
    vs = np.concatenate([np.linspace(-8, 8, 113), [-1e-3, 1e-3, -0.5, 0.5, 3.0, -3.0, 1e-8, 20.0]])
    ref = torch.nn.functional.gelu(torch.tensor(vs, dtype=torch.float64), approximate="tanh").numpy()
    for v, r in zip(vs, ref):
        assert oracle.gelu(v, 1) == pytest.approx(r, rel=1e-13, abs=1e-300), v


def test_gelu_tanh_form_properties():
    # odd-symmetric part: g(v) - g(-v) = v for both forms (1 + s(v), s odd)
    for v in np.linspace(-5, 5, 41):
        assert oracle.gelu(v, 1) - oracle.gelu(-v, 1) == pytest.approx(v, abs=1e-14)
    # the tanh form tracks the exact GeLU to within 1e-3 everywhere and is exact at 0
    vs = np.linspace(-6, 6, 241)
    diff = max(abs(oracle.gelu(v, 1) - _gelu_ref(v)) for v in vs)
    assert 1e-5 < diff < 1e-3
    assert oracle.gelu(0.0, 1) == 0.0


# ---------------------------------------------------------------- closed forms -----------

def _readout_params(W, H, dh, lam_value, ba, bx):
    return dict(
        conv_w=np.tile(np.array([0, 0, 0, 1], np.float32)[:, None], (1, W)),   # identity tap
        conv_b=np.zeros(W, np.float32),
        w_a=np.zeros((H, dh, dh), np.float32), w_x=np.zeros((H, dh, dh), np.float32),
        b_a=np.full(W, ba, np.float32), b_x=np.full(W, bx, np.float32),
        lam=np.asarray(lam_value, np.float32) * np.ones(W, np.float32),
    )


def test_closed_form_geometric_sum():
    """W_a = W_x = 0, identity conv, constant input x0: constant gates give
    h_t = a^(t+1) h0 + beta i x0 (1 - a^(t+1)) / (1 - a)."""
    rng = np.random.default_rng(1)
    B, T, H, dh = 2, 40, 2, 8
    W = H * dh
    lam = rng.uniform(-1.0, 6.0, size=W).astype(np.float32)
    p = _readout_params(W, H, dh, 0.0, 0.0, 0.0)
    p["lam"] = lam
    p["b_a"] = rng.uniform(-2, 2, W).astype(np.float32)
    p["b_x"] = rng.uniform(-2, 2, W).astype(np.float32)
    x0 = rng.standard_normal((B, 1, W)).astype(np.float32)
    x = np.repeat(x0, T, axis=1)
    y = rng.standard_normal((B, T, W)).astype(np.float32)
    h0 = rng.standard_normal((B, W))
    out, hT, _ = oracle.prefill(p, x, y, H, h0=h0, tail0=np.repeat(x0, 3, axis=1))

    r = 1 / (1 + np.exp(-p["b_a"].astype(np.float64)))
    i = 1 / (1 + np.exp(-p["b_x"].astype(np.float64)))
    a = np.power(1 / (1 + np.exp(-lam.astype(np.float64))), C * r)      # a^(c r), power form
    beta = np.sqrt(1 - a * a)
    t = np.arange(T)[None, :, None] + 1
    h = a ** t * h0[:, None, :] + beta * i * x0 * (1 - a ** t) / (1 - a)
    np.testing.assert_allclose(out, h * _gelu_ref(y), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(hT, h[:, -1], rtol=1e-11)


def test_freeze_when_recurrence_gate_is_zero():
    """r_t = 0 => a_t = 1 and sqrt(1 - a_t^2) = 0, so h_t = h_{t-1} exactly, for any input."""
    rng = np.random.default_rng(2)
    B, T, H, dh = 2, 33, 3, 16
    W = H * dh
    p = _params(W, H, dh, rng)
    p["b_a"] = np.full(W, -1e4, np.float32)          # sigma(-1e4) underflows to exactly 0
    x = rng.standard_normal((B, T, W)).astype(np.float32)
    y = rng.standard_normal((B, T, W)).astype(np.float32)
    h0 = rng.standard_normal((B, W))
    out, hT, _ = oracle.prefill(p, x, y, H, h0=h0)
    assert np.array_equal(hT, h0)
    np.testing.assert_allclose(out, h0[:, None, :] * _gelu_ref(y), rtol=1e-13, atol=1e-300)
    _, a_t = oracle.prefill_unit_decay(p, x, y, H, 0, 1)
    assert np.all(a_t == 1.0)


def test_decay_strictly_inside_unit_interval():
    """a = sigma(Lambda) in (0, 1) and a_t = a^(c r_t) with r_t in (0, 1): 0 < a_t < 1."""
    wl = inputs.WORKLOADS["tiny_f32"]
    prob = inputs.make_problem(wl, seed=0)
    for b, hd in [(0, 0), (0, 3)]:
        _, a_t = oracle.prefill_unit_decay(prob.params, prob.x, prob.y, wl.heads, b, hd)
        assert np.all(a_t > 0) and np.all(a_t < 1)
        # and a_t >= a^c (r <= 1): the decay never exceeds its base rate
        lam = prob.params["lam"][hd * wl.head_dim:(hd + 1) * wl.head_dim].astype(np.float64)
        a_c = (1 / (1 + np.exp(-lam))) ** C
        assert np.all(a_t >= a_c[None, :] * (1 - 1e-12))


def test_variance_preservation():
    """i_t = 1, identity conv, x iid N(0,1), constant a_t, unit-variance start:
    Var(h_t) = a^2 Var(h_{t-1}) + (1 - a^2) = 1 for every t (checked within 5 sigma)."""
    rng = np.random.default_rng(3)
    B, T, H, dh = 1, 24, 2048, 16
    W = H * dh
    p = _readout_params(W, H, dh, 2.0, 0.0, 40.0)   # sigma(40) == 1.0 in fp64
    x = rng.standard_normal((B, T, W)).astype(np.float32)
    y = np.full((B, T, W), 8.0, np.float32)
    h0 = rng.standard_normal((B, W))
    out, _, _ = oracle.prefill(p, x, y, H, h0=h0)
    h = out / _gelu_ref(8.0)
    var = (h[0] ** 2).mean(axis=1)                  # over 32768 channels
    sigma = math.sqrt(2.0 / W)
    assert np.all(np.abs(var - 1.0) < 5 * sigma), var
    # from zero state: E[h_t^2] = 1 - a^(2(t+1))
    out0, _, _ = oracle.prefill(p, x, y, H)
    h = out0 / _gelu_ref(8.0)
    r = 0.5
    a = (1 / (1 + math.exp(-2.0))) ** (C * r)
    expect = 1 - a ** (2 * (np.arange(T) + 1))
    var = (h[0] ** 2).mean(axis=1)
    assert np.all(np.abs(var - expect) < 5 * expect * math.sqrt(2.0 / W)), (var, expect)


# ---------------------------------------------------------------- brute force ------------

def _brute_force(p, x, y, H, h0, tail0, reset=None):
    """Independent restatement: torch conv1d over [history, x], dense block-diagonal gate
    matrices, power-form decay, sqrt(1 - a^2), and the unrolled double sum
    h_t = (prod_{s<=t} a_s) h0 + sum_{s<=t} (prod_{s<k<=t} a_k) u_s."""
    B, T, W = x.shape
    xf = inputs.as_f32(x).astype(np.float64)
    yf = inputs.as_f32(y).astype(np.float64)
    seq = torch.from_numpy(np.concatenate([tail0, xf], axis=1)).permute(0, 2, 1)  # [B, W, T+3]
    wt = torch.from_numpy(p["conv_w"].astype(np.float64).T[:, None, :])           # [W, 1, 4]
    xc = torch.nn.functional.conv1d(seq, wt, bias=torch.from_numpy(p["conv_b"].astype(np.float64)),
                                    groups=W).permute(0, 2, 1).numpy()           # [B, T, W]
    wa = inputs.as_f32(p["w_a"]).astype(np.float64)
    wx = inputs.as_f32(p["w_x"]).astype(np.float64)
    Wa = scipy.linalg.block_diag(*wa)
    Wx = scipy.linalg.block_diag(*wx)
    ga = xc @ Wa + p["b_a"].astype(np.float64)
    gx = xc @ Wx + p["b_x"].astype(np.float64)
    r = 1 / (1 + np.exp(-ga))
    i = 1 / (1 + np.exp(-gx))
    a_base = 1 / (1 + np.exp(-p["lam"].astype(np.float64)))
    a = np.power(a_base, C * r)
    u = np.sqrt(1 - a * a) * i * xc
    h = np.zeros((B, T, W))
    for t in range(T):
        acc = np.prod(a[:, :t + 1], axis=1) * h0
        for s in range(t + 1):
            acc = acc + np.prod(a[:, s + 1:t + 1], axis=1) * u[:, s]
        h[:, t] = acc
    return h * _gelu_ref(yf), h[:, -1]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_bruteforce_unrolling_T8(dtype):
    rng = np.random.default_rng(4)
    B, T, H, dh = 2, 8, 3, 8
    W = H * dh
    p = _params(W, H, dh, rng, dtype=dtype)
    x = rng.standard_normal((B, T, W)).astype(np.float32)
    y = rng.standard_normal((B, T, W)).astype(np.float32)
    if dtype == "bf16":
        x, y = inputs.f32_to_bf16_bits(x), inputs.f32_to_bf16_bits(y)
    h0 = rng.standard_normal((B, W))
    tail0 = rng.standard_normal((B, 3, W)).astype(np.float32)
    out, hT, tail = oracle.prefill(p, x, y, H, h0=h0, tail0=tail0)
    ref, ref_h = _brute_force(p, x, y, H, h0, tail0.astype(np.float64))
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(hT, ref_h, rtol=1e-10, atol=1e-12)
    # the carried conv history is the last three raw x-branch inputs, oldest first
    np.testing.assert_array_equal(tail, inputs.as_f32(x)[:, -3:].astype(np.float64))


def test_gate_orientation_is_in_major():
    """gate_o = sum_i xc_i W[i][o]: swapping W for its transpose must change the result."""
    rng = np.random.default_rng(5)
    B, T, H, dh = 1, 6, 2, 8
    W = H * dh
    p = _params(W, H, dh, rng)
    x = rng.standard_normal((B, T, W)).astype(np.float32)
    y = rng.standard_normal((B, T, W)).astype(np.float32)
    out, _, _ = oracle.prefill(p, x, y, H)
    ref, _ = _brute_force(p, x, y, H, np.zeros((B, W)), np.zeros((B, 3, W)))
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)
    pt = dict(p, w_a=np.ascontiguousarray(p["w_a"].transpose(0, 2, 1)),
              w_x=np.ascontiguousarray(p["w_x"].transpose(0, 2, 1)))
    out_t, _, _ = oracle.prefill(pt, x, y, H)
    assert np.max(np.abs(out_t - ref)) > 1e-3


# ---------------------------------------------------------------- conv taps --------------

def _conv_readout(conv_w, conv_b, x, tail0=None):
    """Expose xc: a_t ~ 0 (Lambda = -30, r = 1), i = 1, beta = 1, so h_t = xc_t, and
    y = 8 makes out_t = xc_t * GeLU(8)."""
    B, T, W = x.shape
    p = _readout_params(W, 1, W, -30.0, 40.0, 40.0)
    p["conv_w"], p["conv_b"] = conv_w, conv_b
    y = np.full((B, T, W), 8.0, np.float32)
    out, _, _ = oracle.prefill(p, x, y, 1, tail0=tail0)
    return out / _gelu_ref(8.0)


def test_conv_identity_and_single_taps():
    rng = np.random.default_rng(6)
    B, T, W = 2, 12, 8
    x = rng.standard_normal((B, T, W)).astype(np.float32)
    zb = np.zeros(W, np.float32)
    for k in range(4):
        w = np.zeros((4, W), np.float32)
        w[k] = 1.0
        xc = _conv_readout(w, zb, x)
        shift = 3 - k                          # tap k reads x_{t-3+k}
        expect = np.zeros_like(xc)
        expect[:, shift:] = x[:, :T - shift]
        np.testing.assert_allclose(xc, expect, rtol=1e-14, atol=1e-14)


def test_conv_matches_torch_conv1d_listing_form():
    """The listing: Conv1d(groups=W, kernel 4, padding 3, bias) truncated to the first T."""
    rng = np.random.default_rng(7)
    B, T, W = 2, 17, 8
    x = rng.standard_normal((B, T, W)).astype(np.float32)
    w = rng.standard_normal((4, W)).astype(np.float32)
    bias = rng.standard_normal(W).astype(np.float32)
    xc = _conv_readout(w, bias, x)
    conv = torch.nn.Conv1d(W, W, 4, padding=3, groups=W, bias=True).double()
    with torch.no_grad():
        conv.weight.copy_(torch.from_numpy(w.T[:, None, :].astype(np.float64)))
        conv.bias.copy_(torch.from_numpy(bias.astype(np.float64)))
        ref = conv(torch.from_numpy(x.astype(np.float64)).permute(0, 2, 1))[:, :, :T]
    np.testing.assert_allclose(xc, ref.permute(0, 2, 1).numpy(), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- resets / carry ---------

def test_packed_rows_equal_separate_documents():
    rng = np.random.default_rng(8)
    T, H, dh = 50, 2, 8
    W = H * dh
    p = _params(W, H, dh, rng)
    x = rng.standard_normal((1, T, W)).astype(np.float32)
    y = rng.standard_normal((1, T, W)).astype(np.float32)
    starts = [0, 7, 8, 30, 49]
    reset = np.zeros((1, T), np.uint8)
    reset[0, starts] = 1
    h0 = rng.standard_normal((1, W))
    tail0 = rng.standard_normal((1, 3, W)).astype(np.float32)
    out, hT, tail = oracle.prefill(p, x, y, H, reset=reset, h0=h0, tail0=tail0)
    bounds = starts + [T]
    for s, e in zip(bounds[:-1], bounds[1:]):
        o, hh, tt = oracle.prefill(p, x[:, s:e], y[:, s:e], H)
        np.testing.assert_array_equal(out[:, s:e], o)
    np.testing.assert_array_equal(hT, hh)
    np.testing.assert_array_equal(tail, tt)


def test_reset_cuts_all_dependence_on_the_past():
    rng = np.random.default_rng(9)
    T, H, dh, t0 = 24, 2, 8, 11
    W = H * dh
    p = _params(W, H, dh, rng)
    x = rng.standard_normal((1, T, W)).astype(np.float32)
    y = rng.standard_normal((1, T, W)).astype(np.float32)
    reset = np.zeros((1, T), np.uint8)
    reset[0, t0] = 1
    out1, _, _ = oracle.prefill(p, x, y, H, reset=reset, h0=rng.standard_normal((1, W)))
    x2 = x.copy()
    x2[:, :t0] = rng.standard_normal((1, t0, W))
    out2, _, _ = oracle.prefill(p, x2, y, H, reset=reset, h0=rng.standard_normal((1, W)))
    np.testing.assert_array_equal(out1[:, t0:], out2[:, t0:])
    assert np.max(np.abs(out1[:, :t0] - out2[:, :t0])) > 1e-3


def test_split_prefill_equals_whole():
    rng = np.random.default_rng(10)
    B, T, H, dh, T1 = 2, 20, 2, 8, 7
    W = H * dh
    p = _params(W, H, dh, rng)
    x = inputs.f32_to_bf16_bits(rng.standard_normal((B, T, W)).astype(np.float32))
    y = inputs.f32_to_bf16_bits(rng.standard_normal((B, T, W)).astype(np.float32))
    p["w_a"] = inputs.f32_to_bf16_bits(p["w_a"])
    p["w_x"] = inputs.f32_to_bf16_bits(p["w_x"])
    out, hT, tail = oracle.prefill(p, x, y, H)
    o1, h1, t1 = oracle.prefill(p, x[:, :T1], y[:, :T1], H)
    o2, h2, t2 = oracle.prefill(p, x[:, T1:], y[:, T1:], H, h0=h1, tail0=t1)
    np.testing.assert_array_equal(out, np.concatenate([o1, o2], axis=1))
    np.testing.assert_array_equal(hT, h2)
    np.testing.assert_array_equal(tail, t2)


def test_decode_steps_equal_prefill():
    rng = np.random.default_rng(11)
    B, T, H, dh = 3, 9, 2, 8
    W = H * dh
    p = _params(W, H, dh, rng)
    x = rng.standard_normal((B, T, W)).astype(np.float32)
    y = rng.standard_normal((B, T, W)).astype(np.float32)
    h0 = rng.standard_normal((B, W))
    tail0 = rng.standard_normal((B, 3, W)).astype(np.float32)
    reset = np.zeros((B, T), np.uint8)
    reset[1, 4] = 1
    out, hT, tailT = oracle.prefill(p, x, y, H, reset=reset, h0=h0, tail0=tail0)
    h = h0.copy()
    tail = tail0.astype(np.float64)
    for t in range(T):
        o = oracle.decode(p, x[:, t], y[:, t], H, h, tail, reset=reset[:, t])
        np.testing.assert_array_equal(o, out[:, t])
    np.testing.assert_array_equal(h, hT)
    np.testing.assert_array_equal(tail, tailT)


# ---------------------------------------------------------------- page facts -------------

def test_page_constants_fixture():
    """tests/golden/page_facts.json: constants and worked identities the pages print."""
    with open(os.path.join(GOLDEN, "page_facts.json")) as f:
        facts = json.load(f)
    assert facts["c"] == inputs.C_CONST == C
    assert facts["conv_width"] == inputs.CONV_WIDTH
    lo, hi = facts["a_pow_c_init_range"]
    wl = inputs.WORKLOADS["tiny_f32"]
    prob = inputs.make_problem(wl)
    a = 1 / (1 + np.exp(-prob.params["lam"].astype(np.float64)))
    assert np.all(a ** C >= lo - 1e-6) and np.all(a ** C <= hi + 1e-6)
    # "a_t^2 + (1 - a_t^2) = 1": the squared weights of the update sum to one
    for a_t in facts["variance_identity_examples"]:
        assert a_t ** 2 + (math.sqrt(1 - a_t ** 2)) ** 2 == pytest.approx(1.0, abs=1e-15)


def test_oracle_regression_golden():
    """The oracle still reproduces tests/golden/oracle_small_cases.json bit for bit."""
    from tests.golden import make_golden
    with open(os.path.join(GOLDEN, "oracle_small_cases.json")) as f:
        stored = json.load(f)["cases"]
    for case in stored:
        _, _, out, h, _ = make_golden.make_case(case)
        np.testing.assert_array_equal(out.ravel(), np.array(case["out"]))
        np.testing.assert_array_equal(h.ravel(), np.array(case["h"]))


def test_prefill_units_matches_full_batch():
    """The per-sequence entry point computes exactly what the batched one does."""
    rng = np.random.default_rng(12)
    B, T, H, dh = 3, 30, 3, 8
    W = H * dh
    p = _params(W, H, dh, rng, dtype="bf16")
    x = inputs.f32_to_bf16_bits(rng.standard_normal((B, T, W)).astype(np.float32))
    y = inputs.f32_to_bf16_bits(rng.standard_normal((B, T, W)).astype(np.float32))
    reset = (rng.random((B, T)) < 0.1).astype(np.uint8)
    h0 = rng.standard_normal((B, W))
    tail0 = inputs.f32_to_bf16_bits(rng.standard_normal((B, 3, W)).astype(np.float32))
    out, hT, tT = oracle.prefill(p, x, y, H, reset=reset, h0=h0, tail0=tail0)
    units = [(0, 2), (2, 0), (1, 1)]
    got = oracle.prefill_units(p, x, y, H, units, reset=reset, h0=h0, tail0=tail0)
    for (b, hd), (o, h, t) in got.items():
        sl = slice(hd * dh, (hd + 1) * dh)
        np.testing.assert_array_equal(o, out[b, :, sl])
        np.testing.assert_array_equal(h, hT[b, sl])
        np.testing.assert_array_equal(t, tT[b, :, sl])
