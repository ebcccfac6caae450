"""Pins of the local sliding-window MQA oracle (oracle/mqa.py), by things other than itself:
closed forms of the window, an independent complex-number form of the rotation, the relative
position property of RoPE, dense masked attention through scipy's softmax for a window that
covers the whole sequence, and decode through the ring buffer equal to the prefill; planted
mistakes (an off-by-one window, a flipped rotation, a ring slot off by one) are caught."""

import os

import numpy as np
import pytest
import scipy.special

from oracle import mqa


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_window_of_one_returns_the_token_value():
    q, k, v = _rand((2, 9, 3, 8), 0), _rand((2, 9, 8), 1), _rand((2, 9, 8), 2)
    y = mqa.prefill(q, k, v, window=1)
    for h in range(3):
        np.testing.assert_allclose(y[:, :, h], v, rtol=0, atol=1e-15)


@pytest.mark.parametrize("window", [1, 3, 5, 50])
def test_zero_queries_average_the_window(window):
    T = 11
    q = np.zeros((1, T, 2, 8))
    k, v = _rand((1, T, 8), 3), _rand((1, T, 8), 4)
    y = mqa.prefill(q, k, v, window=window)
    for t in range(T):
        lo = max(0, t - window + 1)
        np.testing.assert_allclose(y[0, t, 0], v[0, lo:t + 1].mean(axis=0), atol=1e-14)


def test_rope_matches_complex_rotation():
    x = _rand((5, 16), 5)
    pos = np.arange(5) * 7 + 3
    got = mqa.rope(x, pos)
    d, half = 16, 8
    z = x[:, :half] + 1j * x[:, half:]
    theta = 10000.0 ** (-2.0 * np.arange(half) / d)
    rz = z * np.exp(1j * pos[:, None] * theta)
    np.testing.assert_allclose(got, np.concatenate([rz.real, rz.imag], axis=1), atol=1e-13)


def test_rope_scores_depend_only_on_relative_position():
    q, k = _rand(32, 6), _rand(32, 7)
    for m, n in ((5, 2), (40, 40), (3, 17)):
        a = mqa.rope(q, np.array(m)) @ mqa.rope(k, np.array(n))
        b = mqa.rope(q, np.array(m + 123)) @ mqa.rope(k, np.array(n + 123))
        assert a == pytest.approx(b, rel=1e-11, abs=1e-12)
    np.testing.assert_allclose(np.linalg.norm(mqa.rope(q, np.array(9))), np.linalg.norm(q), rtol=1e-14)


def test_full_window_is_dense_causal_attention():
    B, T, H, d = 2, 13, 3, 8
    q, k, v = _rand((B, T, H, d), 8), _rand((B, T, d), 9), _rand((B, T, d), 10)
    y = mqa.prefill(q, k, v, window=T + 4, pos0=5)
    pos = 5 + np.arange(T)
    qr = mqa.rope(q, pos[None, :, None])
    kr = mqa.rope(k, pos[None, :])
    mask = np.tril(np.ones((T, T), bool))
    for b in range(B):
        for h in range(H):
            s = (qr[b, :, h] @ kr[b].T) / np.sqrt(d)
            s = np.where(mask, s, -np.inf)
            np.testing.assert_allclose(y[b, :, h], scipy.special.softmax(s, axis=1) @ v[b], atol=1e-12)


def test_ring_buffer_decode_equals_prefill():
    T, H, d, w = 23, 2, 8, 6
    q, k, v = _rand((1, T, H, d), 11), _rand((1, T, d), 12), _rand((1, T, d), 13)
    y = mqa.prefill(q, k, v, window=w)
    cache = mqa.RingCache(w, d)
    for t in range(T):
        np.testing.assert_allclose(mqa.decode_step(cache, q[0, t], k[0, t], v[0, t], t), y[0, t], atol=1e-13)


MUTANTS = {
    "window_one_too_wide": ("lo = max(0, t - window + 1)", "lo = max(0, t - window)"),
    "rotation_sign": ("x1 * c - x2 * s, x2 * c + x1 * s", "x1 * c + x2 * s, x2 * c - x1 * s"),
    "ring_slot_off_by_one": ("self.k[pos % self.w] = k_rot", "self.k[(pos + 1) % self.w] = k_rot"),
}
PINS = [test_window_of_one_returns_the_token_value, lambda: test_zero_queries_average_the_window(3),
        test_rope_matches_complex_rotation, test_full_window_is_dense_causal_attention,
        test_ring_buffer_decode_equals_prefill]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    old, new = MUTANTS[name]
    src = open(os.path.join(os.path.dirname(mqa.__file__), "mqa.py")).read()
    assert src.count(old) == 1
    ns = {"__name__": "mqa_mutant"}
    exec(compile(src.replace(old, new), "mqa_mutant", "exec"), ns)
    for fn in ("prefill", "rope", "decode_step", "RingCache"):
        monkeypatch.setattr(mqa, fn, ns[fn])
    failed = 0
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed, f"no pin caught {name}"
