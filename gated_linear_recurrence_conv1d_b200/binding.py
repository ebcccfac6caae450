"""Thin ctypes binding of librglru.so (argument marshalling only).

Every computation happens in the CUDA library; this module only turns torch tensors into the
device pointers, sizes and structs that ``include/rglru.h`` declares, and raises
:class:`RglruError` on a non-OK status.  PyTorch supplies device memory and the stream.
There is no CPU path: if the library is missing and cannot be built, loading raises.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from . import build as _build

RGLRU_OK = 0
RGLRU_ERR_CUDA = 4
RGLRU_ERR_TIMEOUT = 5
RGLRU_ERR_DEVICE = 6
RGLRU_F32, RGLRU_BF16 = 0, 1
FLAG_GENERIC = 1
FLAG_TEST_WITHHOLD = 2

STATUS_NAMES = {0: "RGLRU_OK", 1: "RGLRU_ERR_INVALID_ARG", 2: "RGLRU_ERR_UNSUPPORTED",
                3: "RGLRU_ERR_WORKSPACE", 4: "RGLRU_ERR_CUDA", 5: "RGLRU_ERR_TIMEOUT",
                6: "RGLRU_ERR_DEVICE"}

EXPORTED = ("rglru_state_init", "rglru_prefill_workspace_size", "rglru_block_prefill",
            "rglru_decode_workspace_size", "rglru_block_decode", "rglru_read_device_status",
            "rglru_status_string", "rglru_abi_version", "rglru_prefill_plan", "rglru_decode_plan",
            "rglru_block_prefill_noalloc", "rglru_last_cuda_error", "rglru_backward_workspace_size",
            "rglru_block_backward", "rglru_backward_plan", "rglru_decode_steps_workspace_size",
            "rglru_block_decode_steps", "rglru_decode_steps_plan", "rglru_layer_workspace_size",
            "rglru_layer_forward", "rglru_layer_plan", "rglru_mqa_workspace_size", "rglru_mqa_prefill",
            "rglru_mqa_decode")

# Fields of rglru_grads, in order (fp32 device tensors).
GRAD_FIELDS = ("dx", "dy", "dh0", "dtail0", "dconv_w", "dconv_b", "dw_a", "dw_x", "db_a", "db_x",
               "dlambda")

# Bytes of the static device scratch behind rglru_block_prefill_noalloc.
NOALLOC_SCRATCH_BYTES = 16 << 20


class RglruError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}{detail}")


class Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("seq_len", ctypes.c_int), ("heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("conv_width", ctypes.c_int),
                ("act_dtype", ctypes.c_int), ("c", ctypes.c_float), ("gelu_tanh", ctypes.c_int),
                ("flags", ctypes.c_uint)]


class Params(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("conv_w", "conv_b", "w_a", "w_x", "b_a", "b_x",
                                                "lambda_")]


class State(ctypes.Structure):
    _fields_ = [("h", ctypes.c_void_p), ("conv_tail", ctypes.c_void_p)]


class Projections(ctypes.Structure):
    _fields_ = [("model_dim", ctypes.c_int), ("w_in_x", ctypes.c_void_p), ("w_in_y", ctypes.c_void_p),
                ("w_out", ctypes.c_void_p)]


class MqaDims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("seq_len", ctypes.c_int), ("q_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("window", ctypes.c_int), ("scale", ctypes.c_float),
                ("rope_base", ctypes.c_float)]


class Grads(ctypes.Structure):
    _fields_ = [(k, ctypes.c_void_p) for k in GRAD_FIELDS]


_lib = None


def library_path() -> str:
    return _build.LIB


def load(build_if_missing: bool = True):
    """Open librglru.so (building it in-tree with nvcc when it is missing or stale)."""
    global _lib
    if _lib is not None:
        return _lib
    path = _build.LIB
    if build_if_missing and _build.stale():
        _build.build()
    if not os.path.exists(path):
        raise RuntimeError(f"librglru.so not found at {path}; build it with "
                           "`python -m gated_linear_recurrence_conv1d_b200.build`")
    lib = ctypes.CDLL(path)
    V, S, I = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    PD, PP, PS = ctypes.POINTER(Dims), ctypes.POINTER(Params), ctypes.POINTER(State)
    lib.rglru_state_init.argtypes = [PD, PS, V]
    lib.rglru_state_init.restype = I
    lib.rglru_prefill_workspace_size.argtypes = [PD]
    lib.rglru_prefill_workspace_size.restype = S
    lib.rglru_decode_workspace_size.argtypes = [PD]
    lib.rglru_decode_workspace_size.restype = S
    lib.rglru_block_prefill.argtypes = [PD, PP, V, V, V, PS, V, V, S, V]
    lib.rglru_block_prefill.restype = I
    lib.rglru_block_prefill_noalloc.argtypes = [PD, PP, V, V, V, PS, V, V, V]
    lib.rglru_block_prefill_noalloc.restype = I
    lib.rglru_block_decode.argtypes = [PD, PP, V, V, V, PS, V, V, S, V]
    lib.rglru_block_decode.restype = I
    lib.rglru_read_device_status.argtypes = [V, S, V]
    lib.rglru_read_device_status.restype = I
    lib.rglru_status_string.argtypes = [I]
    lib.rglru_status_string.restype = ctypes.c_char_p
    PI = ctypes.POINTER(ctypes.c_int)
    lib.rglru_prefill_plan.argtypes = [PD, PI, PI]
    lib.rglru_prefill_plan.restype = I
    lib.rglru_decode_plan.argtypes = [PD, PI, PI]
    lib.rglru_decode_plan.restype = I
    lib.rglru_backward_plan.argtypes = [PD, PI, PI]
    lib.rglru_backward_plan.restype = I
    PG = ctypes.POINTER(Grads)
    lib.rglru_backward_workspace_size.argtypes = [PD]
    lib.rglru_backward_workspace_size.restype = S
    lib.rglru_block_backward.argtypes = [PD, PP, V, V, V, PS, V, V, V, PG, V, S, V]
    lib.rglru_block_backward.restype = I
    lib.rglru_decode_steps_workspace_size.argtypes = [PD, I]
    lib.rglru_decode_steps_workspace_size.restype = S
    lib.rglru_block_decode_steps.argtypes = [PD, PP, V, V, V, I, PS, V, V, S, V]
    lib.rglru_block_decode_steps.restype = I
    lib.rglru_decode_steps_plan.argtypes = [PD, I, PI, PI]
    lib.rglru_decode_steps_plan.restype = I
    PJ = ctypes.POINTER(Projections)
    lib.rglru_layer_workspace_size.argtypes = [PD]
    lib.rglru_layer_workspace_size.restype = S
    lib.rglru_layer_forward.argtypes = [PD, PP, PJ, V, V, PS, V, V, S, V]
    lib.rglru_layer_forward.restype = I
    lib.rglru_layer_plan.argtypes = [PD, PJ, PI, PI]
    lib.rglru_layer_plan.restype = I
    PM = ctypes.POINTER(MqaDims)
    lib.rglru_mqa_workspace_size.argtypes = [PM, I]
    lib.rglru_mqa_workspace_size.restype = S
    lib.rglru_mqa_prefill.argtypes = [PM, V, V, V, I, V, V, V, S, V]
    lib.rglru_mqa_prefill.restype = I
    lib.rglru_mqa_decode.argtypes = [PM, V, V, V, V, V, V, V, S, V]
    lib.rglru_mqa_decode.restype = I
    lib.rglru_last_cuda_error.argtypes = [ctypes.POINTER(ctypes.c_char_p)]
    lib.rglru_last_cuda_error.restype = I
    lib.rglru_abi_version.argtypes = []
    lib.rglru_abi_version.restype = I
    _lib = lib
    return lib


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to the RG-LRU library must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return RGLRU_F32
    if t.dtype == torch.bfloat16:
        return RGLRU_BF16
    raise ValueError(f"unsupported activation dtype {t.dtype}")


def make_dims(batch: int, seq_len: int, heads: int, head_dim: int, act_dtype: int, c: float = 8.0,
              gelu_tanh: int = 0, flags: int = 0) -> Dims:
    return Dims(batch, seq_len, heads, head_dim, 4, act_dtype, c, gelu_tanh, flags)


def make_params(p: dict) -> Params:
    """p: dict of device tensors conv_w, conv_b, w_a, w_x, b_a, b_x, lam (biases may be None)."""
    return Params(*(_ptr(p.get(k)) for k in ("conv_w", "conv_b", "w_a", "w_x", "b_a", "b_x", "lam")))


def last_cuda_error() -> tuple:
    """(cudaError_t value, its name) behind this thread's most recent RGLRU_ERR_CUDA."""
    name = ctypes.c_char_p()
    code = load().rglru_last_cuda_error(ctypes.byref(name))
    return code, (name.value or b"").decode()


def _check(status: int, where: str):
    if status != RGLRU_OK:
        detail = ""
        if status == RGLRU_ERR_CUDA:
            code, name = last_cuda_error()
            detail = f" ({name}, {code})"
        raise RglruError(status, where, detail)


def prefill_workspace_size(dims: Dims) -> int:
    return load().rglru_prefill_workspace_size(ctypes.byref(dims))


def decode_workspace_size(dims: Dims) -> int:
    return load().rglru_decode_workspace_size(ctypes.byref(dims))


def alloc_workspace(nbytes: int, device=None) -> torch.Tensor:
    """Zeroed device workspace (torch allocations are 256-byte aligned)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


def state_init(dims: Dims, h: torch.Tensor, conv_tail: torch.Tensor, stream=None):
    st = State(_ptr(h), _ptr(conv_tail))
    _check(load().rglru_state_init(ctypes.byref(dims), ctypes.byref(st), _stream(stream)),
           "rglru_state_init")


def block_prefill(dims: Dims, params: Params, x: torch.Tensor, y: torch.Tensor,
                  out: torch.Tensor, workspace: torch.Tensor, reset: Optional[torch.Tensor] = None,
                  h: Optional[torch.Tensor] = None, conv_tail: Optional[torch.Tensor] = None,
                  stream=None):
    st = State(_ptr(h), _ptr(conv_tail)) if h is not None else None
    rc = load().rglru_block_prefill(ctypes.byref(dims), ctypes.byref(params), _ptr(x), _ptr(y),
                                    _ptr(reset), ctypes.byref(st) if st is not None else None,
                                    _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "rglru_block_prefill")


def block_prefill_noalloc(dims: Dims, params: Params, x: torch.Tensor, y: torch.Tensor,
                          out: torch.Tensor, reset: Optional[torch.Tensor] = None,
                          h: Optional[torch.Tensor] = None, conv_tail: Optional[torch.Tensor] = None,
                          status_out: Optional[torch.Tensor] = None, stream=None):
    """rglru_block_prefill without a workspace: the library's static device scratch is used
    (for callers that cannot allocate device memory).  status_out: optional 16-byte device
    buffer that receives the device status word after the kernel."""
    st = State(_ptr(h), _ptr(conv_tail)) if h is not None else None
    rc = load().rglru_block_prefill_noalloc(ctypes.byref(dims), ctypes.byref(params), _ptr(x),
                                            _ptr(y), _ptr(reset),
                                            ctypes.byref(st) if st is not None else None,
                                            _ptr(out), _ptr(status_out), _stream(stream))
    _check(rc, "rglru_block_prefill_noalloc")


def block_decode(dims: Dims, params: Params, x: torch.Tensor, y: torch.Tensor, out: torch.Tensor,
                 h: torch.Tensor, conv_tail: torch.Tensor, workspace: torch.Tensor,
                 reset: Optional[torch.Tensor] = None, stream=None):
    st = State(_ptr(h), _ptr(conv_tail))
    rc = load().rglru_block_decode(ctypes.byref(dims), ctypes.byref(params), _ptr(x), _ptr(y),
                                   _ptr(reset), ctypes.byref(st), _ptr(out), _ptr(workspace),
                                   workspace.numel(), _stream(stream))
    _check(rc, "rglru_block_decode")


def decode_steps_workspace_size(dims: Dims, steps: int) -> int:
    return load().rglru_decode_steps_workspace_size(ctypes.byref(dims), int(steps))


def block_decode_steps(dims: Dims, params: Params, x: torch.Tensor, y: torch.Tensor, out: torch.Tensor,
                       h: torch.Tensor, conv_tail: torch.Tensor, workspace: torch.Tensor,
                       reset: Optional[torch.Tensor] = None, stream=None):
    """rglru_block_decode_steps: x, y, out [steps, B, W]; reset [steps, B] uint8 or None."""
    steps = x.shape[0]
    st = State(_ptr(h), _ptr(conv_tail))
    rc = load().rglru_block_decode_steps(ctypes.byref(dims), ctypes.byref(params), _ptr(x), _ptr(y),
                                         _ptr(reset), int(steps), ctypes.byref(st), _ptr(out),
                                         _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "rglru_block_decode_steps")


def decode_steps_plan(dims: Dims, steps: int):
    k, n = ctypes.c_int(), ctypes.c_int()
    fn = load().rglru_decode_steps_plan
    _check(fn(ctypes.byref(dims), int(steps), ctypes.byref(k), ctypes.byref(n)), "rglru_decode_steps_plan")
    return k.value, n.value


def make_projections(model_dim: int, w_in_x: torch.Tensor, w_in_y: torch.Tensor, w_out: torch.Tensor) -> Projections:
    """w_in_x, w_in_y [D, W] and w_out [W, D] device tensors in the act dtype."""
    return Projections(int(model_dim), _ptr(w_in_x), _ptr(w_in_y), _ptr(w_out))


def layer_workspace_size(dims: Dims) -> int:
    return load().rglru_layer_workspace_size(ctypes.byref(dims))


def layer_forward(dims: Dims, params: Params, proj: Projections, u: torch.Tensor, out: torch.Tensor,
                  workspace: torch.Tensor, reset: Optional[torch.Tensor] = None,
                  h: Optional[torch.Tensor] = None, conv_tail: Optional[torch.Tensor] = None, stream=None):
    """rglru_layer_forward: u, out [B, T, D]."""
    st = State(_ptr(h), _ptr(conv_tail)) if h is not None else None
    rc = load().rglru_layer_forward(ctypes.byref(dims), ctypes.byref(params), ctypes.byref(proj), _ptr(u),
                                    _ptr(reset), ctypes.byref(st) if st is not None else None, _ptr(out),
                                    _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "rglru_layer_forward")


def layer_plan(dims: Dims, proj: Projections):
    k, n = ctypes.c_int(), ctypes.c_int()
    _check(load().rglru_layer_plan(ctypes.byref(dims), ctypes.byref(proj), ctypes.byref(k), ctypes.byref(n)),
           "rglru_layer_plan")
    return k.value, n.value


def make_mqa_dims(batch: int, seq_len: int, q_heads: int, head_dim: int, window: int, scale: Optional[float] = None,
                  rope_base: float = 10000.0) -> MqaDims:
    return MqaDims(batch, seq_len, q_heads, head_dim, window,
                   (head_dim ** -0.5) if scale is None else scale, rope_base)


def mqa_workspace_size(dims: MqaDims, decode: bool = False) -> int:
    return load().rglru_mqa_workspace_size(ctypes.byref(dims), int(decode))


def mqa_prefill(dims: MqaDims, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                workspace: torch.Tensor, pos0: int = 0, cache: Optional[torch.Tensor] = None, stream=None):
    """rglru_mqa_prefill: q [B, T, H, d], k, v [B, T, d] -> out [B, T, H, d]."""
    rc = load().rglru_mqa_prefill(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), int(pos0), _ptr(out), _ptr(cache),
                                  _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "rglru_mqa_prefill")


def mqa_decode(dims: MqaDims, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, pos: torch.Tensor,
               cache: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor, stream=None):
    """rglru_mqa_decode: q [B, H, d], k, v [B, d], pos [B] int32 (device) -> out [B, H, d]."""
    rc = load().rglru_mqa_decode(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(pos), _ptr(cache), _ptr(out),
                                 _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "rglru_mqa_decode")


def backward_workspace_size(dims: Dims) -> int:
    return load().rglru_backward_workspace_size(ctypes.byref(dims))


def block_backward(dims: Dims, params: Params, x: torch.Tensor, y: torch.Tensor,
                   dout: torch.Tensor, grads: dict, workspace: torch.Tensor,
                   reset: Optional[torch.Tensor] = None, h0: Optional[torch.Tensor] = None,
                   tail0: Optional[torch.Tensor] = None, dh_final: Optional[torch.Tensor] = None,
                   dtail_final: Optional[torch.Tensor] = None, stream=None):
    """rglru_block_backward: writes the gradients into the fp32 tensors of ``grads`` (keys of
    GRAD_FIELDS; dh0 / dtail0 may be absent)."""
    st = State(_ptr(h0), _ptr(tail0)) if h0 is not None else None
    g = Grads(*(_ptr(grads.get(k)) for k in GRAD_FIELDS))
    rc = load().rglru_block_backward(ctypes.byref(dims), ctypes.byref(params), _ptr(x), _ptr(y),
                                     _ptr(reset), ctypes.byref(st) if st is not None else None,
                                     _ptr(dout), _ptr(dh_final), _ptr(dtail_final), ctypes.byref(g),
                                     _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "rglru_block_backward")


def _plan(fn, dims: Dims):
    k, n = ctypes.c_int(), ctypes.c_int()
    _check(fn(ctypes.byref(dims), ctypes.byref(k), ctypes.byref(n)), fn.__name__)
    return k.value, n.value


def prefill_plan(dims: Dims):
    """(kernel kind, launches per call) of rglru_block_prefill for these dims."""
    return _plan(load().rglru_prefill_plan, dims)


def decode_plan(dims: Dims):
    return _plan(load().rglru_decode_plan, dims)


def prefill_launches(dims: Dims) -> int:
    return prefill_plan(dims)[1]


def decode_launches(dims: Dims) -> int:
    return decode_plan(dims)[1]


def backward_plan(dims: Dims):
    return _plan(load().rglru_backward_plan, dims)


def backward_launches(dims: Dims) -> int:
    return backward_plan(dims)[1]


def read_device_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device status code."""
    return load().rglru_read_device_status(_ptr(workspace), workspace.numel(), _stream(stream))


class RGLRUBlock:
    """Convenience wrapper holding device parameters for one block.

    params: dict of numpy arrays as made by ``inputs.make_params`` (bf16 as uint16 bits).
    """

    def __init__(self, params: dict, heads: int, head_dim: int, act: str, device="cuda",
                 c: float = 8.0, gelu_tanh: int = 0, flags: int = 0):
        self.heads, self.head_dim, self.c, self.gelu_tanh, self.flags = heads, head_dim, c, gelu_tanh, flags
        self.act = act
        self.act_code = RGLRU_BF16 if act == "bf16" else RGLRU_F32
        self.device = device
        self.tensors = {k: to_device(v, device) for k, v in params.items() if v is not None}
        self.params = make_params(self.tensors)

    def dims(self, batch: int, seq_len: int) -> Dims:
        return make_dims(batch, seq_len, self.heads, self.head_dim, self.act_code, self.c,
                         self.gelu_tanh, self.flags)


def to_device(a, device="cuda") -> torch.Tensor:
    """numpy -> device tensor; uint16 arrays are bf16 bit patterns."""
    import numpy as np
    if isinstance(a, torch.Tensor):
        return a.to(device)
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(a).to(device)


def to_numpy_act(t: torch.Tensor):
    """device tensor -> numpy (bf16 as uint16 bits, fp32 as float32)."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view("uint16")
    return t.numpy()
