"""Parity at the full workload sizes, in the launch configuration bench.py times.

The GPU runs the whole workload; the fp64 oracle recomputes a sample of whole sequences
((batch row, head) pairs, every token, or every decode step of sampled rows) and the two are
compared element by element under the parity bar of tests/gpu_util.py.  Sequences are
independent (block-diagonal gates, per-channel conv and recurrence), so a sampled sequence is
checked exactly as if the oracle had run the whole batch.
"""

import numpy as np
import pytest
import torch

import oracle
from gated_linear_recurrence_conv1d_b200 import binding, inputs
from tests.gpu_util import GpuProblem, assert_close, to_np

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

WL = inputs.WORKLOADS


def _check_units(prob, out, h, tail, units):
    wl = prob.wl
    dh = wl.head_dim
    refs = oracle.prefill_units(prob.params, prob.x, prob.y, wl.heads, units, reset=prob.reset,
                                h0=prob.h0, tail0=prob.tail0)
    for (b, hd), (ref, ref_h, ref_tail) in refs.items():
        sl = slice(hd * dh, (hd + 1) * dh)
        assert_close(to_np(out[b, :, sl]), ref, wl.dtype, f"{wl.name} unit ({b},{hd}) out")
        if h is not None:
            assert_close(to_np(h[b, sl]), ref_h, wl.dtype, f"{wl.name} unit ({b},{hd}) h")
            np.testing.assert_array_equal(to_np(tail[b, :, sl]), ref_tail)


@pytest.mark.parametrize("name,units", [
    ("rg2b_bf16", [(0, 0), (3, 5), (7, 9)]),
    ("long_bf16", [(0, 0), (0, 15)]),
    ("packed_bf16", [(0, 0), (9, 11), (15, 23)]),
])
def test_full_size_prefill_sampled_sequences(name, units):
    prob = inputs.make_problem(WL[name], seed=0)
    gp = GpuProblem(prob)
    out, h, tail, status = gp.prefill(use_state=True)
    assert status == binding.RGLRU_OK
    torch.cuda.synchronize()
    _check_units(prob, out, h, tail, units)


def test_full_size_decode_sampled_rows():
    """1024 decode steps of the batch-256 workload; rows 0, 101 and 255 (all heads) are
    replayed by the oracle and compared at every step, and the final state at the end."""
    wl = WL["decode_bf16"]
    prob = inputs.make_problem(wl, seed=0)
    gp = GpuProblem(prob)
    B = wl.batch
    h, tail = gp.new_state(B)
    dims = gp.block.dims(B, 1)
    ws = binding.alloc_workspace(binding.decode_workspace_size(dims))
    rows = np.array([0, 101, 255])
    h_ref = prob.h0[rows].astype(np.float64).copy()
    t_ref = oracle.tail_from_act(prob.tail0[rows]).copy()
    out = torch.empty_like(gp.x)
    for s in range(wl.decode_steps):
        binding.block_decode(dims, gp.block.params, gp.x[s], gp.y[s], out[s], h, tail, ws)
    assert binding.read_device_status(ws) == binding.RGLRU_OK
    outs = to_np(out[:, rows])
    for s in range(wl.decode_steps):
        ref = oracle.decode(prob.params, prob.x[s][rows], prob.y[s][rows], wl.heads, h_ref, t_ref)
        assert_close(outs[s], ref, "bf16", f"decode step {s}")
    assert_close(to_np(h[rows]), h_ref, "bf16", "decode final h")
    np.testing.assert_array_equal(to_np(tail[rows]), t_ref)
