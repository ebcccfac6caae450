"""The block with its projections (rglru_layer_forward) against the fp64 layer oracle, and
against the same computation assembled from torch matmuls and rglru_block_prefill."""

import numpy as np
import pytest
import torch

import oracle
from gated_linear_recurrence_conv1d_b200 import binding, inputs
from tests.gpu_util import assert_close, rel_err, to_np

pytestmark = pytest.mark.gpu


def _problem(B, T, H, D, seed, resets=True, state=True):
    base = inputs.WORKLOADS["packed_bf16"] if resets else inputs.WORKLOADS["rg2b_bf16"]
    kw = dict(doc_len=(8, 90)) if resets else {}
    wl = base.scaled(batch=B, seq_len=T, heads=H, random_state=state, **kw)
    prob = inputs.make_problem(wl, seed=seed)
    rng = np.random.default_rng(seed + 3)
    W = wl.width
    u = inputs.f32_to_bf16_bits(rng.standard_normal((B, T, D)).astype(np.float32))
    proj = {"w_in_x": inputs.f32_to_bf16_bits((rng.standard_normal((D, W)) / np.sqrt(D)).astype(np.float32)),
            "w_in_y": inputs.f32_to_bf16_bits((rng.standard_normal((D, W)) / np.sqrt(D)).astype(np.float32)),
            "w_out": inputs.f32_to_bf16_bits((rng.standard_normal((W, D)) / np.sqrt(W)).astype(np.float32))}
    return wl, prob, u, proj


@pytest.mark.parametrize("B,T,H,D", [(2, 100, 2, 384), (1, 64, 1, 256), (3, 37, 2, 192)])
def test_layer_matches_oracle(B, T, H, D):
    wl, prob, u, proj = _problem(B, T, H, D, seed=80 + T)
    dev = "cuda"
    block = binding.RGLRUBlock(prob.params, wl.heads, wl.head_dim, "bf16", dev)
    pt = {k: binding.to_device(v, dev) for k, v in proj.items()}
    pj = binding.make_projections(D, pt["w_in_x"], pt["w_in_y"], pt["w_out"])
    dims = block.dims(B, T)
    assert binding.layer_plan(dims, pj)[0] == 1
    ud = binding.to_device(u, dev)
    out = torch.empty(B, T, D, dtype=torch.bfloat16, device=dev)
    h = binding.to_device(prob.h0, dev).clone()
    tail = binding.to_device(prob.tail0, dev).clone()
    reset = None if prob.reset is None else binding.to_device(prob.reset, dev)
    ws = binding.alloc_workspace(binding.layer_workspace_size(dims), dev)
    binding.layer_forward(dims, block.params, pj, ud, out, ws, reset=reset, h=h, conv_tail=tail)
    assert binding.read_device_status(ws) == binding.RGLRU_OK
    # the layer oracle at the block's bf16 interface: x, y and z rounded where they cross it
    ref, ref_h, _, _ = oracle.layer(prob.params, proj, u, wl.heads, reset=prob.reset, h0=prob.h0, tail0=prob.tail0,
                                    act_interface=True)
    assert_close(to_np(out), ref, "bf16", "layer out")
    assert_close(to_np(h), ref_h, "bf16", "layer h")

    # the same from torch matmuls (fp32 accumulation, bf16 results) around the block
    x = torch.matmul(ud.float(), pt["w_in_x"].float()).to(torch.bfloat16)
    y = torch.matmul(ud.float(), pt["w_in_y"].float()).to(torch.bfloat16)
    z = torch.empty_like(x)
    h2 = binding.to_device(prob.h0, dev).clone()
    t2 = binding.to_device(prob.tail0, dev).clone()
    wsb = binding.alloc_workspace(binding.prefill_workspace_size(dims), dev)
    binding.block_prefill(dims, block.params, x, y, z, wsb, reset=reset, h=h2, conv_tail=t2)
    o2 = torch.matmul(z.float(), pt["w_out"].float()).to(torch.bfloat16)
    assert rel_err(to_np(out), to_np(o2)) <= 1e-2
    # the tail holds the last projected inputs; the two projections accumulate in different
    # orders, so an element may round to the neighbouring bf16 value (one ulp, 2^-7 relative)
    np.testing.assert_allclose(to_np(tail), to_np(t2), rtol=2.0 ** -7, atol=0)
