"""Tensor-core prefill specifics: it is the path taken for bf16 / head_dim 256, it agrees with
the portable kernels and with the oracle across chunk, look-back and reset boundaries, and its
bounded waits turn a withheld carry into RGLRU_ERR_TIMEOUT without hanging the GPU.
"""

import numpy as np
import pytest
import torch

import oracle
from gated_linear_recurrence_conv1d_b200 import binding, inputs
from tests.gpu_util import GpuProblem, assert_close, rel_err, to_np

pytestmark = pytest.mark.gpu

BASE = inputs.WORKLOADS


def test_plan_uses_tensor_cores_for_bf16_dh256():
    d = binding.make_dims(8, 2048, 10, 256, binding.RGLRU_BF16)
    kind, launches = binding.prefill_plan(d)
    assert kind == 1 and launches >= 1
    d.flags = binding.FLAG_GENERIC
    assert binding.prefill_plan(d)[0] == 0
    assert binding.prefill_plan(binding.make_dims(1, 256, 4, 64, binding.RGLRU_F32))[0] == 0


@pytest.mark.parametrize("B,T,H", [(1, 64, 1), (2, 65, 2), (3, 1000, 3), (1, 5000, 2), (16, 130, 1)])
def test_fused_matches_oracle_and_generic(B, T, H):
    wl = BASE["rg2b_bf16"].scaled(batch=B, seq_len=T, heads=H, random_state=True)
    prob = inputs.make_problem(wl, seed=100 + T)
    gp = GpuProblem(prob)
    out, h, tail, status = gp.prefill()
    assert status == binding.RGLRU_OK
    ref, ref_h, ref_tail = oracle.prefill(prob.params, prob.x, prob.y, H, h0=prob.h0, tail0=prob.tail0)
    assert_close(to_np(out), ref, "bf16", "fused out")
    assert_close(to_np(h), ref_h, "bf16", "fused h")
    np.testing.assert_array_equal(to_np(tail), ref_tail)
    gen = GpuProblem(prob, flags=binding.FLAG_GENERIC)
    out_g, h_g, _, _ = gen.prefill()
    assert rel_err(to_np(out), to_np(out_g)) <= 1e-2
    assert rel_err(to_np(h), to_np(h_g)) <= 1e-2


def test_fused_long_sequence_lookback_chain():
    """One row, many 64-token chunks spread over the CTAs of each group: the carry crosses
    CTAs through the look-back on every chunk boundary."""
    wl = BASE["long_bf16"].scaled(batch=1, seq_len=20000, heads=1)
    prob = inputs.make_problem(wl, seed=7)
    gp = GpuProblem(prob)
    out, h, _, status = gp.prefill()
    assert status == binding.RGLRU_OK
    ref, ref_h, _ = oracle.prefill(prob.params, prob.x, prob.y, 1)
    assert_close(to_np(out), ref, "bf16", "long out")
    assert_close(to_np(h), ref_h, "bf16", "long h")


def test_fused_packed_resets():
    wl = BASE["packed_bf16"].scaled(batch=4, seq_len=3000, heads=2, doc_len=(20, 700),
                                    random_state=True)
    prob = inputs.make_problem(wl, seed=12)
    gp = GpuProblem(prob)
    out, h, tail, status = gp.prefill()
    assert status == binding.RGLRU_OK
    ref, ref_h, ref_tail = oracle.prefill(prob.params, prob.x, prob.y, 2, reset=prob.reset,
                                          h0=prob.h0, tail0=prob.tail0)
    assert_close(to_np(out), ref, "bf16", "packed out")
    assert_close(to_np(h), ref_h, "bf16", "packed h")
    np.testing.assert_array_equal(to_np(tail), ref_tail)


def test_fused_no_state_and_tanh_gelu():
    wl = BASE["rg2b_bf16"].scaled(batch=2, seq_len=333, heads=2, gelu_tanh=1)
    prob = inputs.make_problem(wl, seed=13)
    gp = GpuProblem(prob)
    out, _, _, status = gp.prefill(use_state=False)
    assert status == binding.RGLRU_OK
    ref, _, _ = oracle.prefill(prob.params, prob.x, prob.y, 2, gelu_tanh=1)
    assert_close(to_np(out), ref, "bf16", "tanh gelu out")


def test_fused_bitwise_repeatable():
    wl = BASE["packed_bf16"].scaled(batch=3, seq_len=2500, heads=2, doc_len=(30, 900))
    prob = inputs.make_problem(wl, seed=14)
    gp = GpuProblem(prob)
    a, _, _, _ = gp.prefill(use_state=False)
    for _ in range(3):
        b, _, _, _ = gp.prefill(use_state=False)
        assert torch.equal(a, b)


def test_withheld_carry_times_out_and_context_survives():
    """Test hook: the first chunk of group 0 never publishes its carry, so its successor's
    bounded wait expires; the kernel must report RGLRU_ERR_TIMEOUT and return, and the same
    context must run a normal prefill afterwards."""
    wl = BASE["rg2b_bf16"].scaled(batch=1, seq_len=64 * 8, heads=1)
    prob = inputs.make_problem(wl, seed=15)
    gp = GpuProblem(prob)
    _, _, _, status = gp.prefill(use_state=False, flags=binding.FLAG_TEST_WITHHOLD)
    assert status == binding.RGLRU_ERR_TIMEOUT
    out, _, _, status = gp.prefill(use_state=False)
    assert status == binding.RGLRU_OK
    ref, _, _ = oracle.prefill(prob.params, prob.x, prob.y, 1)
    assert_close(to_np(out), ref, "bf16", "after timeout")


def test_fused_nonzero_biases_resets_and_state():
    """Gate biases (folded into the tensor-memory accumulators), a conv bias, resets and a
    carried state together, against the oracle and the portable kernels."""
    wl = BASE["packed_bf16"].scaled(batch=2, seq_len=700, heads=2, doc_len=(30, 400),
                                    random_state=True)
    prob = inputs.make_problem(wl, seed=21)
    rng = np.random.default_rng(21)
    W = wl.width
    for k in ("b_a", "b_x", "conv_b"):
        prob.params[k] = (0.7 * rng.standard_normal(W)).astype(np.float32)
    gp = GpuProblem(prob)
    out, h, tail, status = gp.prefill()
    assert status == binding.RGLRU_OK
    ref, ref_h, ref_tail = oracle.prefill(prob.params, prob.x, prob.y, wl.heads, reset=prob.reset,
                                          h0=prob.h0, tail0=prob.tail0)
    assert_close(to_np(out), ref, "bf16", "biased out")
    assert_close(to_np(h), ref_h, "bf16", "biased h")
    np.testing.assert_array_equal(to_np(tail), ref_tail)


def test_fused_closed_recurrence_gate_freezes_state():
    """b_a = -1e4 makes r_t = 0, so a_t = 1 and sqrt(1 - a_t^2) = 0: the carried state passes
    through every token unchanged and out_t = h_0 GeLU(y_t)."""
    wl = BASE["rg2b_bf16"].scaled(batch=2, seq_len=200, heads=2, random_state=True)
    prob = inputs.make_problem(wl, seed=22)
    prob.params["b_a"] = np.full(wl.width, -1e4, np.float32)
    gp = GpuProblem(prob)
    out, h, _, status = gp.prefill()
    assert status == binding.RGLRU_OK
    ref, ref_h, _ = oracle.prefill(prob.params, prob.x, prob.y, wl.heads, h0=prob.h0, tail0=prob.tail0)
    np.testing.assert_array_equal(ref_h, prob.h0.astype(np.float64))     # the oracle's freeze
    assert_close(to_np(out), ref, "bf16", "frozen out")
    assert rel_err(to_np(h), ref_h) <= 1e-6


def test_plan_uses_tensor_cores_for_decode_bf16_dh256():
    d = binding.make_dims(256, 1, 10, 256, binding.RGLRU_BF16)
    kind, launches = binding.decode_plan(d)
    assert kind == 1 and launches == 1
    assert binding.decode_workspace_size(d) >= 256
    d.flags = binding.FLAG_GENERIC
    assert binding.decode_plan(d)[0] == 0


@pytest.mark.parametrize("B", [1, 77, 130, 256])
def test_tensor_decode_matches_oracle_and_generic(B):
    """Row tiles of 128 with a ragged last tile; biases and resets; against the oracle and the
    portable kernel over a few steps."""
    wl = BASE["decode_bf16"].scaled(batch=B, heads=2, decode_steps=4)
    prob = inputs.make_problem(wl, seed=30 + B)
    rng = np.random.default_rng(B)
    for k in ("b_a", "b_x", "conv_b"):
        prob.params[k] = (0.5 * rng.standard_normal(wl.width)).astype(np.float32)
    outs = {}
    for flags in (0, binding.FLAG_GENERIC):
        gp = GpuProblem(prob, flags=flags)
        h, tail = gp.new_state(B)
        dims = gp.block.dims(B, 1)
        ws = binding.alloc_workspace(binding.decode_workspace_size(dims))
        h_ref = prob.h0.astype(np.float64).copy()
        t_ref = oracle.tail_from_act(prob.tail0).copy()
        res = []
        for s in range(4):
            rst_np = (np.arange(B) % 5 == s).astype(np.uint8)
            out = torch.empty_like(gp.x[s])
            binding.block_decode(dims, gp.block.params, gp.x[s], gp.y[s], out, h, tail, ws,
                                 reset=binding.to_device(rst_np))
            ref = oracle.decode(prob.params, prob.x[s], prob.y[s], wl.heads, h_ref, t_ref, reset=rst_np)
            assert_close(to_np(out), ref, "bf16", f"decode step {s} flags {flags}")
            np.testing.assert_array_equal(to_np(tail), t_ref)
            res.append(to_np(out))
        assert binding.read_device_status(ws) == binding.RGLRU_OK
        assert_close(to_np(h), h_ref, "bf16", "decode h")
        outs[flags] = np.stack(res)
    assert rel_err(outs[0], outs[binding.FLAG_GENERIC]) <= 1e-2


def test_tensor_decode_withheld_block_times_out_and_context_survives():
    """Test hook: the decode step's first CTA keeps its conv block from the other CTAs of its
    cluster, so their bounded waits expire; the call must report RGLRU_ERR_TIMEOUT and return,
    and the same context must then run a correct decode step."""
    B = 130
    wl = BASE["decode_bf16"].scaled(batch=B, heads=2, decode_steps=1)
    prob = inputs.make_problem(wl, seed=44)
    bad = GpuProblem(prob, flags=binding.FLAG_TEST_WITHHOLD)
    h, tail = bad.new_state(B)
    dims = bad.block.dims(B, 1)
    assert binding.decode_plan(dims) == (1, 1)
    ws = binding.alloc_workspace(binding.decode_workspace_size(dims))
    out = torch.empty_like(bad.x[0])
    binding.block_decode(dims, bad.block.params, bad.x[0], bad.y[0], out, h, tail, ws)
    assert binding.read_device_status(ws) == binding.RGLRU_ERR_TIMEOUT

    gp = GpuProblem(prob)
    h, tail = gp.new_state(B)
    dims = gp.block.dims(B, 1)
    binding.block_decode(dims, gp.block.params, gp.x[0], gp.y[0], out, h, tail, ws)
    assert binding.read_device_status(ws) == binding.RGLRU_OK
    h_ref = prob.h0.astype(np.float64).copy()
    t_ref = oracle.tail_from_act(prob.tail0).copy()
    ref = oracle.decode(prob.params, prob.x[0], prob.y[0], wl.heads, h_ref, t_ref)
    assert_close(to_np(out), ref, "bf16", "decode after timeout")
    assert_close(to_np(h), h_ref, "bf16", "decode h after timeout")
    np.testing.assert_array_equal(to_np(tail), t_ref)

