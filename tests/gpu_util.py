"""Helpers for the GPU parity tests: run the CUDA path through the C ABI, compare with the
fp64 oracle under the error metrics of the parity bar.

1. The bar: max relative error in the max norm, rel = max_i |g_i - r_i| / max_i |r_i|, at most
   1e-5 for fp32 inputs and 2e-2 for bf16 inputs with fp32 state.
2. RMS relative error, rms(g - r) / rms(r), at most 2e-6 (fp32) / 5e-3 (bf16): it catches a
   bias spread over many elements that the max norm would let through.
3. Element-wise error, max_i |g_i - r_i| / max(|r_i|, 0.1 rms(r)) (the denominator floored where
   h_t * GeLU(y_t) crosses zero): at most 2e-2 for bf16, the same bar element by element.  For
   fp32 it is 1e-4: there the floor amplifies plain rounding, and an exact fp32 emulation of
   the block already scores 4e-5.  The bf16 kernels round only the tensor-core operand of the
   gate contraction to bf16; the conv output entering the state update stays fp32.
"""

from __future__ import annotations

import numpy as np
import torch

from gated_linear_recurrence_conv1d_b200 import binding, inputs

TOL = {"f32": 1e-5, "bf16": 2e-2}
TOL_RMS = {"f32": 2e-6, "bf16": 5e-3}
TOL_ELEMENTWISE = {"f32": 1e-4, "bf16": 2e-2}


def rel_err(g: np.ndarray, r: np.ndarray) -> float:
    """Primary metric: max-norm relative error."""
    g = np.asarray(g, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    if r.size == 0:
        return 0.0
    return float(np.max(np.abs(g - r)) / max(float(np.max(np.abs(r))), 1e-300))


def rel_err_elementwise(g: np.ndarray, r: np.ndarray) -> float:
    """Secondary guard: element-wise relative error with the denominator floored at 0.1 RMS."""
    g = np.asarray(g, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    if r.size == 0:
        return 0.0
    floor = 0.1 * float(np.sqrt(np.mean(r * r)))
    den = np.maximum(np.abs(r), max(floor, 1e-300))
    return float(np.max(np.abs(g - r) / den))


def rel_err_rms(g: np.ndarray, r: np.ndarray) -> float:
    g = np.asarray(g, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    if r.size == 0:
        return 0.0
    return float(np.sqrt(np.mean((g - r) ** 2)) / max(float(np.sqrt(np.mean(r * r))), 1e-300))


def assert_close(g, r, dtype: str, what: str = ""):
    e = rel_err(g, r)
    e_rms = rel_err_rms(g, r)
    e2 = rel_err_elementwise(g, r)
    assert e <= TOL[dtype], f"{what}: max-norm relative error {e:.3e} > {TOL[dtype]}"
    assert e_rms <= TOL_RMS[dtype], f"{what}: RMS relative error {e_rms:.3e} > {TOL_RMS[dtype]}"
    assert e2 <= TOL_ELEMENTWISE[dtype], f"{what}: element-wise error {e2:.3e} > {TOL_ELEMENTWISE[dtype]}"
    return e, e2


def act_to_f64(a: np.ndarray) -> np.ndarray:
    return inputs.as_f32(a).astype(np.float64)


class GpuProblem:
    """A problem uploaded to the device, run through the C ABI."""

    def __init__(self, prob: inputs.Problem, flags: int = 0, device="cuda"):
        wl = prob.wl
        self.prob = prob
        self.wl = wl
        self.block = binding.RGLRUBlock(prob.params, wl.heads, wl.head_dim, wl.dtype, device,
                                        gelu_tanh=wl.gelu_tanh, flags=flags)
        self.x = binding.to_device(prob.x, device)
        self.y = binding.to_device(prob.y, device)
        self.reset = None if prob.reset is None else binding.to_device(prob.reset, device)
        self.device = device

    def new_state(self, batch):
        W = self.wl.width
        dt = torch.bfloat16 if self.wl.dtype == "bf16" else torch.float32
        if self.prob.h0 is not None:
            h = binding.to_device(self.prob.h0, self.device).clone()
            tail = binding.to_device(self.prob.tail0, self.device).clone()
        else:
            h = torch.zeros(batch, W, device=self.device)
            tail = torch.zeros(batch, 3, W, device=self.device, dtype=dt)
        return h, tail

    def prefill(self, x=None, y=None, reset=None, state=None, use_state=True, flags=None):
        x = self.x if x is None else x
        y = self.y if y is None else y
        reset = self.reset if reset is None else reset
        B, T = x.shape[0], x.shape[1]
        dims = self.block.dims(B, T)
        if flags is not None:
            dims.flags = flags
        ws = binding.alloc_workspace(binding.prefill_workspace_size(dims), self.device)
        out = torch.empty_like(x)
        h = tail = None
        if use_state:
            h, tail = state if state is not None else self.new_state(B)
        binding.block_prefill(dims, self.block.params, x, y, out, ws, reset=reset, h=h,
                              conv_tail=tail)
        status = binding.read_device_status(ws)
        return out, h, tail, status


def to_np(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return inputs.bf16_bits_to_f32(binding.to_numpy_act(t)).astype(np.float64)
    return t.detach().cpu().double().numpy()
