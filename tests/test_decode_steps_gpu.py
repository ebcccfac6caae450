"""The persistent multi-step decode (rglru_block_decode_steps) against the fp64 oracle stepped
token by token, and against the single-step entry point called once per step.

Continuous batching: reset[s][b] makes slot b start a new sequence at step s; the oracle applies
the same reset before the same step.  The full decode workload (batch 256, 10 heads x 256, 1024
steps) runs in one launch, with three rows replayed by the oracle at every step.
"""

import numpy as np
import pytest
import torch

import oracle
from gated_linear_recurrence_conv1d_b200 import binding, inputs
from tests.gpu_util import GpuProblem, assert_close, rel_err, to_np

pytestmark = pytest.mark.gpu

BASE = inputs.WORKLOADS


def _run_steps(gp, B, steps, reset_np=None):
    h, tail = gp.new_state(B)
    dims = gp.block.dims(B, 1)
    ws = binding.alloc_workspace(binding.decode_steps_workspace_size(dims, steps))
    out = torch.empty_like(gp.x[:steps])
    rst = None if reset_np is None else binding.to_device(np.ascontiguousarray(reset_np))
    binding.block_decode_steps(dims, gp.block.params, gp.x[:steps].contiguous(), gp.y[:steps].contiguous(),
                               out, h, tail, ws, reset=rst)
    assert binding.read_device_status(ws) == binding.RGLRU_OK
    return out, h, tail


@pytest.mark.parametrize("B", [1, 77, 130, 256])
def test_decode_steps_match_oracle_and_single_steps(B):
    steps = 7
    wl = BASE["decode_bf16"].scaled(batch=B, heads=2, decode_steps=steps)
    prob = inputs.make_problem(wl, seed=60 + B)
    rng = np.random.default_rng(B)
    for k in ("b_a", "b_x", "conv_b"):
        prob.params[k] = (0.5 * rng.standard_normal(wl.width)).astype(np.float32)
    reset_np = (rng.random((steps, B)) < 0.2).astype(np.uint8)
    gp = GpuProblem(prob)
    dims = gp.block.dims(B, 1)
    assert binding.decode_steps_plan(dims, steps) == (1, 1)
    out, h, tail = _run_steps(gp, B, steps, reset_np)

    h_ref = prob.h0.astype(np.float64).copy()
    t_ref = oracle.tail_from_act(prob.tail0).copy()
    for s in range(steps):
        ref = oracle.decode(prob.params, prob.x[s], prob.y[s], wl.heads, h_ref, t_ref, reset=reset_np[s])
        assert_close(to_np(out[s]), ref, "bf16", f"multi-step decode, step {s}")
    assert_close(to_np(h), h_ref, "bf16", "multi-step decode h")
    np.testing.assert_array_equal(to_np(tail), t_ref)

    # the same steps through the single-step entry point
    h1, t1 = gp.new_state(B)
    ws = binding.alloc_workspace(binding.decode_workspace_size(dims))
    o1 = torch.empty_like(out)
    for s in range(steps):
        binding.block_decode(dims, gp.block.params, gp.x[s], gp.y[s], o1[s], h1, t1, ws,
                             reset=binding.to_device(np.ascontiguousarray(reset_np[s])))
    assert rel_err(to_np(out), to_np(o1)) <= 1e-2
    np.testing.assert_array_equal(to_np(tail), to_np(t1))


def test_decode_steps_one_step_and_no_resets():
    wl = BASE["decode_bf16"].scaled(batch=20, heads=1, decode_steps=1)
    prob = inputs.make_problem(wl, seed=71)
    gp = GpuProblem(prob)
    out, h, tail = _run_steps(gp, 20, 1)
    h_ref = prob.h0.astype(np.float64).copy()
    t_ref = oracle.tail_from_act(prob.tail0).copy()
    ref = oracle.decode(prob.params, prob.x[0], prob.y[0], 1, h_ref, t_ref)
    assert_close(to_np(out[0]), ref, "bf16", "one step")
    assert_close(to_np(h), h_ref, "bf16", "one step h")
    np.testing.assert_array_equal(to_np(tail), t_ref)


def test_decode_steps_generic_shapes_loop_the_portable_step():
    """fp32 (and other head widths) run the portable step kernel once per step: `steps`
    launches, same results as the oracle."""
    wl = BASE["tiny_f32"].scaled(batch=5, seq_len=1, random_state=True, decode_steps=6)
    prob = inputs.make_problem(wl, seed=72)
    gp = GpuProblem(prob)
    dims = gp.block.dims(5, 1)
    assert binding.decode_steps_plan(dims, 6) == (0, 6)
    out, h, tail = _run_steps(gp, 5, 6)
    h_ref = prob.h0.astype(np.float64).copy()
    t_ref = oracle.tail_from_act(prob.tail0).copy()
    for s in range(6):
        ref = oracle.decode(prob.params, prob.x[s], prob.y[s], wl.heads, h_ref, t_ref)
        assert_close(to_np(out[s]), ref, "f32", f"portable multi-step, step {s}")
    assert_close(to_np(h), h_ref, "f32", "portable multi-step h")


@pytest.mark.slow
def test_full_size_decode_steps_sampled_rows():
    """The decode workload in one launch: 1024 steps of batch 256 x 10 heads x 256 with a
    slot reset every few steps; rows 0, 101 and 255 replayed by the oracle at every step."""
    wl = BASE["decode_bf16"]
    prob = inputs.make_problem(wl, seed=0)
    gp = GpuProblem(prob)
    B, steps = wl.batch, wl.decode_steps
    rng = np.random.default_rng(5)
    reset_np = (rng.random((steps, B)) < 0.01).astype(np.uint8)
    out, h, tail = _run_steps(gp, B, steps, reset_np)
    rows = np.array([0, 101, 255])
    h_ref = prob.h0[rows].astype(np.float64).copy()
    t_ref = oracle.tail_from_act(prob.tail0[rows]).copy()
    outs = to_np(out[:, rows])
    for s in range(steps):
        ref = oracle.decode(prob.params, prob.x[s][rows], prob.y[s][rows], wl.heads, h_ref, t_ref,
                            reset=reset_np[s][rows])
        assert_close(outs[s], ref, "bf16", f"decode step {s}")
    assert_close(to_np(h[rows]), h_ref, "bf16", "final h")
    np.testing.assert_array_equal(to_np(tail[rows]), t_ref)
