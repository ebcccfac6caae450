"""rglru_block_prefill_noalloc: prefill for callers that cannot allocate device memory.

Such callers (an engine whose device memory is one pool carved up before serving, a plugin
inside a host that owns every allocation, code where an allocation would synchronise the
device) cannot hand rglru_block_prefill a workspace.  The no-alloc entry point takes its
scratch from a fixed static area in the library's device image instead.  Its results must be
those of the regular entry point, call after call, although every call reuses the same area
and finds the previous call's contents there.

This file is collected last on purpose: if it fails, a run that stops at the first failure has
already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

from gated_linear_recurrence_conv1d_b200 import binding, inputs
from tests.gpu_util import GpuProblem, assert_close, to_np


def _problem(batch, seq_len, heads, seed):
    """bf16, head_dim 256 (the tensor-core kernel, whose look-back needs scratch), packed
    documents with resets, a random initial state read and written back."""
    wl = inputs.WORKLOADS["packed_bf16"].scaled(batch=batch, seq_len=seq_len, heads=heads,
                                                doc_len=(40, 300), random_state=True)
    return GpuProblem(inputs.make_problem(wl, seed=seed))


def _run_both(gp):
    """(regular entry point's out, h, tail), (no-alloc entry point's out, h, tail, status)."""
    wl = gp.wl
    out_ref, h_ref, tail_ref, status = gp.prefill(use_state=True)
    assert status == binding.RGLRU_OK
    dims = gp.block.dims(wl.batch, wl.seq_len)
    assert binding.prefill_workspace_size(dims) <= binding.NOALLOC_SCRATCH_BYTES
    h, tail = gp.new_state(wl.batch)
    out = torch.empty_like(gp.x)
    status_buf = torch.full((256,), 0xFF, dtype=torch.uint8, device=gp.device)
    binding.block_prefill_noalloc(dims, gp.block.params, gp.x, gp.y, out, reset=gp.reset, h=h,
                                  conv_tail=tail, status_out=status_buf)
    dev_status = binding.read_device_status(status_buf)
    return (out_ref, h_ref, tail_ref), (out, h, tail, dev_status)


def _compare(ref, got, what):
    out_ref, h_ref, tail_ref = ref
    out, h, tail, dev_status = got
    assert dev_status == binding.RGLRU_OK, f"{what}: device status {dev_status}"
    assert_close(to_np(out), to_np(out_ref), "bf16", f"{what} out")
    assert_close(to_np(h), to_np(h_ref), "bf16", f"{what} h")
    np.testing.assert_array_equal(to_np(tail), to_np(tail_ref))


@pytest.mark.gpu
def test_noalloc_prefill_matches_regular_entry_point_twice():
    # two calls in a row through the shared static scratch: the second one, of another shape,
    # finds the first one's tickets, flags and carries in the area
    gp1 = _problem(batch=3, seq_len=1000, heads=2, seed=1)
    _compare(*_run_both(gp1), "first call")
    gp2 = _problem(batch=2, seq_len=777, heads=3, seed=2)
    _compare(*_run_both(gp2), "second call")
    torch.cuda.synchronize()


def test_noalloc_rejects_problems_beyond_the_static_area():
    # host-side check: nothing is enqueued (the pointers below are never dereferenced)
    lib = binding.load()
    fake = 0x10000
    d = binding.make_dims(16, 8192, 24, 256, binding.RGLRU_BF16)
    assert binding.prefill_workspace_size(d) > binding.NOALLOC_SCRATCH_BYTES
    p = binding.Params(*(ctypes.c_void_p(fake) if k in ("conv_w", "w_a", "w_x", "lambda_") else None
                         for k, _ in binding.Params._fields_))
    rc = lib.rglru_block_prefill_noalloc(ctypes.byref(d), ctypes.byref(p), ctypes.c_void_p(fake),
                                         ctypes.c_void_p(fake + 0x100), None, None,
                                         ctypes.c_void_p(fake + 0x200), None, None)
    assert rc == 3                                                  # RGLRU_ERR_WORKSPACE
    assert lib.rglru_status_string(rc).decode().startswith("RGLRU_ERR_WORKSPACE")
