"""Backward pass on the GPU against the fp64 oracle's gradients (every output of
rglru_block_backward, element by element).

The portable kernels compute in fp32 from the exact input values.  The tensor-core path (bf16,
head_dim 256) runs its dense contractions on bf16 operands split into hi + lo parts (fp32 to
about 2^-16), so the same bar serves it and both activation dtypes.  It is ten times the forward's
fp32 bar: the backward chains about three times as many roundings per element (the forward
again, the reverse recurrence, two transposed contractions) and its parameter gradients are
sums over all B T tokens; a wrong term, sign, index or reset gives errors of order one.
"""

import numpy as np
import pytest
import torch

import oracle
from gated_linear_recurrence_conv1d_b200 import binding, inputs
from tests.gpu_util import GpuProblem, rel_err, rel_err_elementwise, rel_err_rms, to_np

pytestmark = pytest.mark.gpu

TOL_MAX, TOL_RMS, TOL_ELEM = 1e-4, 2e-5, 1e-2
KEYS = {"dx": "dx", "dy": "dy", "dh0": "dh0", "dtail0": "dtail0", "dconv_w": "dconv_w",
        "dconv_b": "dconv_b", "dw_a": "dw_a", "dw_x": "dw_x", "db_a": "db_a", "db_x": "db_x",
        "dlambda": "dlam"}


def _run(wl, seed, with_state=True, with_final=True, biases=True):
    prob = inputs.make_problem(wl, seed=seed)
    rng = np.random.default_rng(seed + 7)
    B, T, W, H = wl.batch, wl.seq_len, wl.width, wl.heads
    if biases:
        for k in ("b_a", "b_x", "conv_b"):
            prob.params[k] = (0.5 * rng.standard_normal(W)).astype(np.float32)
    dout = inputs.make_activation(wl, rng, B, T)
    h0 = rng.standard_normal((B, W)).astype(np.float32) if with_state else None
    tail0 = inputs.make_activation(wl, rng, B, 3) if with_state else None
    dhf = rng.standard_normal((B, W)).astype(np.float32) if with_final else None
    dtf = rng.standard_normal((B, 3, W)).astype(np.float32) if with_final else None

    gp = GpuProblem(prob)
    dev = gp.device
    dims = gp.block.dims(B, T)
    ws = binding.alloc_workspace(binding.backward_workspace_size(dims), dev)
    shapes = {"dx": (B, T, W), "dy": (B, T, W), "dh0": (B, W), "dtail0": (B, 3, W),
              "dconv_w": (4, W), "dconv_b": (W,), "dw_a": (H, wl.head_dim, wl.head_dim),
              "dw_x": (H, wl.head_dim, wl.head_dim), "db_a": (W,), "db_x": (W,), "dlambda": (W,)}
    grads = {k: torch.full(s, float("nan"), device=dev, dtype=torch.float32) for k, s in shapes.items()}
    td = lambda a: None if a is None else binding.to_device(a, dev)  # noqa: E731
    binding.block_backward(dims, gp.block.params, gp.x, gp.y, td(dout), grads, ws, reset=gp.reset,
                           h0=td(h0), tail0=td(tail0), dh_final=td(dhf), dtail_final=td(dtf))
    assert binding.read_device_status(ws) == binding.RGLRU_OK
    ref = oracle.backward(prob.params, prob.x, prob.y, H, dout, reset=prob.reset,
                          h0=None if h0 is None else h0.astype(np.float64), tail0=tail0,
                          dh_final=None if dhf is None else dhf.astype(np.float64),
                          dtail_final=None if dtf is None else dtf.astype(np.float64),
                          gelu_tanh=wl.gelu_tanh)
    return grads, ref


def _compare(grads, ref, label):
    for k, rk in KEYS.items():
        g, r = to_np(grads[k]), ref[rk]
        assert np.all(np.isfinite(g)), f"{label} {k}: non-finite values"
        if not np.any(r):
            assert not np.any(g), f"{label} {k}: expected zeros"
            continue
        e, er, ee = rel_err(g, r), rel_err_rms(g, r), rel_err_elementwise(g, r)
        assert e <= TOL_MAX, f"{label} {k}: max-norm relative error {e:.3e}"
        assert er <= TOL_RMS, f"{label} {k}: RMS relative error {er:.3e}"
        assert ee <= TOL_ELEM, f"{label} {k}: element-wise error {ee:.3e}"


@pytest.mark.parametrize("B,T,H,dh,dtype,tanh", [
    (2, 70, 2, 64, "f32", 0),      # two full tiles and a ragged one
    (2, 100, 2, 256, "bf16", 0),   # the tensor-core backward: chunks, a ragged one, resets
    (3, 257, 2, 256, "bf16", 1),   # tanh GeLU, more rows than chunks of the dW slices
    (3, 2, 3, 16, "f32", 0),       # shorter than the conv history
    (1, 45, 2, 48, "f32", 1),      # a head width that does not divide the CTA
])
def test_backward_matches_oracle(B, T, H, dh, dtype, tanh):
    base = inputs.WORKLOADS["packed_bf16"] if T > 8 else inputs.WORKLOADS["tiny_f32"]
    wl = base.scaled(batch=B, seq_len=T, heads=H, head_dim=dh, dtype=dtype, gelu_tanh=tanh,
                     doc_len=(5, 40) if T > 8 else None)
    grads, ref = _run(wl, seed=50 + T)
    _compare(grads, ref, f"B{B} T{T} H{H} dh{dh} {dtype}")


def test_backward_long_carry_across_many_chunks():
    """The tensor-core reverse scan cuts a row into chunks and chains their carries: rows of
    1100 tokens (18 chunks, a ragged last one, more than one prefetch block of chunks) with
    documents of several hundred tokens, so that g crosses many chunk boundaries."""
    wl = inputs.WORKLOADS["packed_bf16"].scaled(batch=2, seq_len=1100, heads=1, doc_len=(300, 900))
    grads, ref = _run(wl, seed=77)
    _compare(grads, ref, "long carry")


def test_backward_without_state_or_final_gradients():
    wl = inputs.WORKLOADS["tiny_f32"].scaled(batch=2, seq_len=40, heads=2, head_dim=32)
    grads, ref = _run(wl, seed=3, with_state=False, with_final=False, biases=False)
    _compare(grads, ref, "zero state")


def test_tensor_backward_agrees_with_portable_and_repeats_bitwise():
    wl = inputs.WORKLOADS["packed_bf16"].scaled(batch=2, seq_len=96, heads=2, doc_len=(10, 60))
    assert binding.backward_plan(binding.make_dims(2, 96, 2, 256, binding.RGLRU_BF16))[0] == 1
    a, ref = _run(wl, seed=21)
    _compare(a, ref, "tensor backward")
    b, _ = _run(wl, seed=21)
    for k in a:
        assert torch.equal(a[k], b[k]), k


def test_backward_bitwise_repeatable():
    wl = inputs.WORKLOADS["tiny_f32"].scaled(batch=2, seq_len=50, heads=2, head_dim=64)
    a, _ = _run(wl, seed=9)
    b, _ = _run(wl, seed=9)
    for k in a:
        assert torch.equal(a[k], b[k]), k
