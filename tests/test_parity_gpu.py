"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle, element by element,
on seeded inputs that span several tiles and a ragged tail, plus edge cases and the
self-consistency identities (split prefill, prefill = decode steps, packed = separate).
"""

import numpy as np
import pytest
import torch

import oracle
from gated_linear_recurrence_conv1d_b200 import binding, inputs
from tests.gpu_util import TOL, GpuProblem, assert_close, rel_err, to_np

pytestmark = pytest.mark.gpu

BASE = inputs.WORKLOADS


def _oracle(prob, reset=None, use_state=True):
    wl = prob.wl
    h0 = prob.h0 if use_state else None
    t0 = prob.tail0 if use_state else None
    return oracle.prefill(prob.params, prob.x, prob.y, wl.heads, reset=reset if reset is not None else prob.reset,
                          h0=h0, tail0=t0, gelu_tanh=wl.gelu_tanh)


def _check_prefill(wl, seed=0, flags=0, use_state=True):
    prob = inputs.make_problem(wl, seed=seed)
    gp = GpuProblem(prob, flags=flags)
    out, h, tail, status = gp.prefill(use_state=use_state)
    assert status == binding.RGLRU_OK
    ref_out, ref_h, ref_tail = _oracle(prob, use_state=use_state)
    e, _ = assert_close(to_np(out), ref_out, wl.dtype, f"{wl.name} out")
    if use_state:
        assert_close(to_np(h), ref_h, wl.dtype, f"{wl.name} state h")
        np.testing.assert_array_equal(to_np(tail), ref_tail)     # conv history: exact copy
    return e


def test_tiny_f32_workload_exact_config():
    """The tiny fp32 workload at its full size: B1 T256 W256 (4 x 64)."""
    _check_prefill(BASE["tiny_f32"], use_state=False)
    _check_prefill(BASE["tiny_f32"], use_state=True)


@pytest.mark.parametrize("dh", [16, 48, 64, 128, 256])
def test_f32_head_dims_ragged(dh):
    wl = BASE["tiny_f32"].scaled(batch=2, seq_len=77, heads=2, head_dim=dh, random_state=True)
    _check_prefill(wl, seed=dh)


@pytest.mark.parametrize("T", [1, 2, 3, 5, 127, 129, 300])
def test_bf16_dh256_ragged_lengths(T):
    wl = BASE["rg2b_bf16"].scaled(batch=2, seq_len=T, heads=2, random_state=True)
    _check_prefill(wl, seed=T)


def test_bf16_long_memory_decay():
    wl = BASE["long_bf16"].scaled(batch=1, seq_len=1000, heads=2)
    _check_prefill(wl, seed=3, use_state=False)


def test_bf16_packed_resets():
    wl = BASE["packed_bf16"].scaled(batch=3, seq_len=600, heads=2, doc_len=(5, 200),
                                    random_state=True)
    _check_prefill(wl, seed=4)


def test_bf16_reset_on_every_token_and_first_token():
    wl = BASE["packed_bf16"].scaled(batch=2, seq_len=40, heads=1, doc_len=(1, 1),
                                    random_state=True)
    _check_prefill(wl, seed=5)


def test_gelu_tanh_variant():
    wl = BASE["rg2b_bf16"].scaled(batch=1, seq_len=64, heads=2, gelu_tanh=1)
    _check_prefill(wl, seed=6, use_state=False)
    wl = BASE["tiny_f32"].scaled(gelu_tanh=1)
    _check_prefill(wl, seed=6, use_state=False)


def test_split_prefill_matches_whole_on_gpu():
    wl = BASE["rg2b_bf16"].scaled(batch=2, seq_len=200, heads=2, random_state=True)
    prob = inputs.make_problem(wl, seed=7)
    gp = GpuProblem(prob)
    out, h, tail, _ = gp.prefill()
    t1 = 83
    h1, tail1 = gp.new_state(2)
    o1, _, _, _ = gp.prefill(x=gp.x[:, :t1].contiguous(), y=gp.y[:, :t1].contiguous(), state=(h1, tail1))
    o2, _, _, _ = gp.prefill(x=gp.x[:, t1:].contiguous(), y=gp.y[:, t1:].contiguous(), state=(h1, tail1))
    whole = to_np(out)
    split = np.concatenate([to_np(o1), to_np(o2)], axis=1)
    assert rel_err(split, whole) <= 1e-2
    assert rel_err(to_np(h1), to_np(h)) <= 1e-3
    np.testing.assert_array_equal(to_np(tail1), to_np(tail))


def _decode_run(wl, steps, seed, flags=0, reset_every=0):
    prob = inputs.make_problem(wl.scaled(decode_steps=steps), seed=seed)
    gp = GpuProblem(prob, flags=flags)
    B = wl.batch
    h, tail = gp.new_state(B)
    dims = gp.block.dims(B, 1)
    ws = binding.alloc_workspace(binding.decode_workspace_size(dims))
    h_ref = prob.h0.astype(np.float64).copy()
    t_ref = oracle.tail_from_act(prob.tail0).copy()
    for s in range(steps):
        rst_np = None
        rst = None
        if reset_every and s % reset_every == reset_every - 1:
            rst_np = (np.arange(B) % 3 == 0).astype(np.uint8)
            rst = binding.to_device(rst_np)
        out = torch.empty_like(gp.x[s])
        binding.block_decode(dims, gp.block.params, gp.x[s], gp.y[s], out, h, tail, ws, reset=rst)
        ref = oracle.decode(prob.params, prob.x[s], prob.y[s], wl.heads, h_ref, t_ref, reset=rst_np,
                            gelu_tanh=wl.gelu_tanh)
        assert_close(to_np(out), ref, wl.dtype, f"decode step {s}")
        np.testing.assert_array_equal(to_np(tail), t_ref)
    assert binding.read_device_status(ws) == binding.RGLRU_OK
    assert_close(to_np(h), h_ref, wl.dtype, "decode final h")


def test_decode_steps_bf16_with_resets():
    wl = BASE["decode_bf16"].scaled(batch=24, heads=2)
    _decode_run(wl, steps=12, seed=8, reset_every=5)


def test_decode_steps_f32():
    wl = BASE["tiny_f32"].scaled(batch=5, seq_len=1, random_state=True)
    _decode_run(wl, steps=10, seed=9)


def test_decode_matches_prefill_on_gpu():
    wl = BASE["rg2b_bf16"].scaled(batch=3, seq_len=16, heads=2, random_state=True)
    prob = inputs.make_problem(wl, seed=10)
    gp = GpuProblem(prob)
    out, h, tail, _ = gp.prefill()
    h2, tail2 = gp.new_state(3)
    dims = gp.block.dims(3, 1)
    ws = binding.alloc_workspace(binding.decode_workspace_size(dims))
    outs = []
    for t in range(16):
        o = torch.empty(3, wl.width, dtype=torch.bfloat16, device="cuda")
        binding.block_decode(dims, gp.block.params, gp.x[:, t].contiguous(), gp.y[:, t].contiguous(),
                             o, h2, tail2, ws)
        outs.append(to_np(o))
    assert rel_err(np.stack(outs, axis=1), to_np(out)) <= 1e-2
    np.testing.assert_array_equal(to_np(tail2), to_np(tail))


def test_state_init_zeroes():
    wl = BASE["rg2b_bf16"].scaled(batch=2, heads=1)
    dims = binding.make_dims(2, 1, 1, 256, binding.RGLRU_BF16)
    h = torch.randn(2, 256, device="cuda")
    tail = torch.randn(2, 3, 256, device="cuda").bfloat16()
    binding.state_init(dims, h, tail)
    torch.cuda.synchronize()
    assert torch.count_nonzero(h) == 0 and torch.count_nonzero(tail.float()) == 0
    del wl


def test_repeat_runs_are_bitwise_identical():
    wl = BASE["packed_bf16"].scaled(batch=2, seq_len=700, heads=2, doc_len=(50, 300))
    prob = inputs.make_problem(wl, seed=11)
    gp = GpuProblem(prob)
    a, _, _, _ = gp.prefill(use_state=False)
    b, _, _, _ = gp.prefill(use_state=False)
    assert torch.equal(a, b)
