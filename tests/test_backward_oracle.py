"""Pins of the oracle's backward pass (CPU only).

The pages give the forward only; the backward is its chain rule.  The oracle's gradients are
pinned against something other than themselves: central finite differences of the forward
oracle, Richardson-extrapolated (error O(h^4)), on inputs placed on a coarse grid so that every
perturbed input is exactly representable in fp32; and closed forms where a gate freezes the
state or a reset cuts the past off.
"""

import numpy as np
import pytest

import oracle

B, T, H, DH = 2, 7, 2, 16
W = H * DH


def _grid(a, step=2.0 ** -12):
    """fp32 values on a grid coarse enough that +-2^-9 perturbations stay exact."""
    return (np.round(a / step) * step).astype(np.float32)


def _problem(seed=0, reset_at=((1, 3),), state=True):
    rng = np.random.default_rng(seed)
    p = dict(conv_w=_grid(rng.standard_normal((4, W)) * 0.5), conv_b=_grid(rng.standard_normal(W) * 0.3),
             w_a=_grid(rng.standard_normal((H, DH, DH)) / 4), w_x=_grid(rng.standard_normal((H, DH, DH)) / 4),
             b_a=_grid(rng.standard_normal(W) * 0.5), b_x=_grid(rng.standard_normal(W) * 0.5),
             lam=_grid(rng.uniform(0.5, 4.0, W)))
    x = _grid(rng.standard_normal((B, T, W)))
    y = _grid(rng.standard_normal((B, T, W)))
    reset = np.zeros((B, T), np.uint8)
    for b, t in reset_at:
        reset[b, t] = 1
    h0 = rng.standard_normal((B, W)) if state else None
    tail0 = _grid(rng.standard_normal((B, 3, W))) if state else None
    dout = _grid(rng.standard_normal((B, T, W)))
    dhf = rng.standard_normal((B, W))
    dtf = rng.standard_normal((B, 3, W))
    return p, x, y, reset, h0, tail0, dout, dhf, dtf


def _loss(p, x, y, reset, h0, tail0, dout, dhf, dtf, gelu_tanh):
    out, h, tail = oracle.prefill(p, x, y, H, reset=reset, h0=h0, tail0=tail0, gelu_tanh=gelu_tanh)
    return (dout.astype(np.float64) * out).sum() + (dhf * h).sum() + (dtf * tail).sum()


def _fd_check(gelu_tanh, seed, per_tensor=4, tol=1e-7):
    p, x, y, reset, h0, tail0, dout, dhf, dtf = _problem(seed)
    g = oracle.backward(p, x, y, H, dout, reset=reset, h0=h0, tail0=tail0, dh_final=dhf,
                        dtail_final=dtf, gelu_tanh=gelu_tanh)
    rng = np.random.default_rng(seed + 100)
    targets = [(x, "dx"), (y, "dy"), (p["conv_w"], "dconv_w"), (p["conv_b"], "dconv_b"),
               (p["w_a"], "dw_a"), (p["w_x"], "dw_x"), (p["b_a"], "db_a"), (p["b_x"], "db_x"),
               (p["lam"], "dlam"), (h0, "dh0"), (tail0, "dtail0")]
    worst = 0.0
    for arr, name in targets:
        for _ in range(per_tensor):
            idx = tuple(int(rng.integers(0, s)) for s in arr.shape)
            base = arr[idx].copy()

            def deriv(step):
                arr[idx] = base + step
                lp = _loss(p, x, y, reset, h0, tail0, dout, dhf, dtf, gelu_tanh)
                arr[idx] = base - step
                lm = _loss(p, x, y, reset, h0, tail0, dout, dhf, dtf, gelu_tanh)
                arr[idx] = base
                return (lp - lm) / (2 * step)

            h = 2.0 ** -8
            fd = (4 * deriv(h / 2) - deriv(h)) / 3
            an = g[name][idx]
            err = abs(fd - an) / max(1e-3, abs(an))
            worst = max(worst, err)
            assert err < tol, f"{name}{idx}: analytic {an!r} vs finite difference {fd!r}"
    return worst


def test_backward_matches_finite_differences():
    _fd_check(gelu_tanh=0, seed=0)


def test_backward_tanh_gelu_matches_finite_differences():
    _fd_check(gelu_tanh=1, seed=1, per_tensor=2)


def test_backward_bf16_inputs_equal_their_fp32_widening():
    p, x, y, reset, h0, tail0, dout, dhf, dtf = _problem(2)
    # bf16 by truncation; the fp32 side then gets exactly the truncated values, widened
    to_bf16 = lambda a: (a.view(np.uint32) >> 16).astype(np.uint16)  # noqa: E731
    pb = dict(p, w_a=to_bf16(p["w_a"]), w_x=to_bf16(p["w_x"]))
    x16, y16, d16, t16 = (to_bf16(_grid(a, 2.0 ** -4)) for a in (x, y, dout, tail0))
    widen = lambda a: (a.astype(np.uint32) << 16).view(np.float32)  # noqa: E731
    pf = dict(p, w_a=widen(pb["w_a"]), w_x=widen(pb["w_x"]))
    g16 = oracle.backward(pb, x16, y16, H, d16, reset=reset, h0=h0, tail0=t16, dh_final=dhf, dtail_final=dtf)
    g32 = oracle.backward(pf, widen(x16), widen(y16), H, widen(d16), reset=reset, h0=h0, tail0=widen(t16),
                          dh_final=dhf, dtail_final=dtf)
    for k in g16:
        np.testing.assert_array_equal(g16[k], g32[k], err_msg=k)


def test_backward_frozen_state_closed_form():
    """b_a = -1e4 makes r = 0 exactly: a = 1, beta = 0, h_t = h_{-1} for every t.  Then
    dL/dh_{-1} = dh_final + sum_t dout_t GeLU(y_t), and nothing reaches x, the gates or Lambda."""
    p, x, y, _, h0, tail0, dout, dhf, _ = _problem(3)
    p["b_a"] = np.full(W, -1e4, np.float32)
    g = oracle.backward(p, x, y, H, dout, h0=h0, tail0=tail0, dh_final=dhf)
    gel = np.vectorize(oracle.gelu)(y.astype(np.float64))
    expect = dhf + (dout.astype(np.float64) * gel).sum(axis=1)
    np.testing.assert_allclose(g["dh0"], expect, rtol=1e-13, atol=1e-13)
    for k in ("dx", "dw_a", "dw_x", "db_a", "db_x", "dlam", "dconv_w", "dconv_b", "dtail0"):
        assert not np.any(g[k]), k


def test_backward_reset_at_the_first_token_cuts_the_initial_state():
    p, x, y, _, h0, tail0, dout, dhf, dtf = _problem(4, reset_at=((0, 0), (1, 0)))
    reset = np.zeros((B, T), np.uint8)
    reset[:, 0] = 1
    g = oracle.backward(p, x, y, H, dout, reset=reset, h0=h0, tail0=tail0, dh_final=dhf, dtail_final=dtf)
    assert not np.any(g["dh0"]) and not np.any(g["dtail0"])


def test_gelu_tanh_derivative_matches_torch_autograd():
    """The backward's tanh-GeLU derivative against torch autograd of torch's own fp64
    gelu(approximate="tanh"): one token per channel, out = h_0 GeLU(y), so
    dy / (dout h_0) = GeLU'(y) for 16 values of y across [-6, 6]."""
    import torch
    vs = np.linspace(-6.0, 6.0, 16).astype(np.float32)
    t = torch.tensor(vs.astype(np.float64), requires_grad=True)
    torch.nn.functional.gelu(t, approximate="tanh").sum().backward()
    ref = t.grad.numpy()
    p = dict(conv_w=np.zeros((4, 16), np.float32), conv_b=np.ones(16, np.float32),
             w_a=np.zeros((1, 16, 16), np.float32), w_x=np.zeros((1, 16, 16), np.float32),
             b_a=np.zeros(16, np.float32), b_x=np.full(16, 40.0, np.float32), lam=np.full(16, 2.0, np.float32))
    x = np.zeros((1, 1, 16), np.float32)
    y = vs.reshape(1, 1, 16)
    dout = np.ones((1, 1, 16), np.float32)
    _, h_after, _ = oracle.prefill(p, x, y, 1, gelu_tanh=1)
    g = oracle.backward(p, x, y, 1, dout, gelu_tanh=1)
    got = g["dy"][0, 0] / h_after[0]
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("v", [-6.0, -1.5, -0.3, 0.0, 0.7, 2.5, 9.0])
@pytest.mark.parametrize("tanh_form", [0, 1])
def test_gelu_derivative_matches_a_difference_quotient(v, tanh_form):
    """One token: out = h_0 GeLU(y), so dy = dout h_0 GeLU'(y); GeLU' is checked against a
    central difference quotient of the oracle's GeLU (h_0 taken from the forward)."""
    step = 1e-5
    fd = (oracle.gelu(v + step, tanh_form) - oracle.gelu(v - step, tanh_form)) / (2 * step)
    p = dict(conv_w=np.zeros((4, 16), np.float32), conv_b=np.ones(16, np.float32),
             w_a=np.zeros((1, 16, 16), np.float32), w_x=np.zeros((1, 16, 16), np.float32),
             b_a=np.zeros(16, np.float32), b_x=np.full(16, 40.0, np.float32), lam=np.full(16, 2.0, np.float32))
    x = np.zeros((1, 1, 16), np.float32)
    y = np.full((1, 1, 16), v, np.float32)
    dout = np.ones((1, 1, 16), np.float32)
    _, h_after, _ = oracle.prefill(p, x, y, 1, h0=np.zeros((1, 16)), tail0=np.zeros((1, 3, 16), np.float32),
                                   gelu_tanh=tanh_form)
    g = oracle.backward(p, x, y, 1, dout, gelu_tanh=tanh_form)
    expect = h_after[0, 0] * fd
    assert h_after[0, 0] > 0.1
    assert abs(g["dy"][0, 0, 0] - expect) <= 1e-8 * max(1.0, abs(expect))
