"""Host-side checks of the C ABI (no GPU needed, nothing is launched).

The library must load on a machine without a GPU, export every entry point that
include/rglru.h declares, and reject bad arguments on the host with the documented codes.
"""

import ctypes
import os
import re

import pytest

from gated_linear_recurrence_conv1d_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "rglru.h")).read()
    return re.findall(r"RGLRU_API\s+[\w\s\*]+?\b(rglru_\w+)\s*\(", src)


def test_library_loads_and_exports_every_declared_symbol():
    lib = binding.load()
    names = _declared()
    assert len(names) >= 8
    assert set(names) == set(binding.EXPORTED)
    for n in names:
        assert getattr(lib, n) is not None
    assert lib.rglru_abi_version() == 1


def test_status_strings():
    lib = binding.load()
    for code, name in binding.STATUS_NAMES.items():
        assert lib.rglru_status_string(code).decode().startswith(name)
    assert lib.rglru_status_string(99).decode() == "RGLRU_ERR_UNKNOWN"


def test_last_cuda_error_starts_clear():
    """A host thread that has had no failed CUDA call reads back cudaSuccess."""
    import threading
    got = []
    t = threading.Thread(target=lambda: got.append(binding.last_cuda_error()))
    t.start()
    t.join()
    assert got == [(0, "cudaSuccess")]


def test_cuda_status_error_carries_the_runtime_error_name():
    with pytest.raises(binding.RglruError, match=r"RGLRU_ERR_CUDA \(cudaSuccess, 0\)"):
        binding._check(binding.RGLRU_ERR_CUDA, "probe")


def _dims(**kw):
    d = dict(batch=2, seq_len=16, heads=2, head_dim=64, act_dtype=binding.RGLRU_BF16)
    d.update(kw)
    return binding.make_dims(**d)


def test_workspace_size_queries():
    assert binding.prefill_workspace_size(_dims()) >= 16
    assert binding.decode_workspace_size(_dims()) >= 16
    assert binding.prefill_workspace_size(_dims(seq_len=0)) == 0
    assert binding.prefill_workspace_size(_dims(head_dim=24)) == 0
    d = _dims()
    d.conv_width = 3
    assert binding.prefill_workspace_size(d) == 0


FAKE = 0x10000  # a 256-aligned non-null address: never dereferenced, validation fails first


def _params(**over):
    p = dict(conv_w=FAKE, conv_b=None, w_a=FAKE, w_x=FAKE, b_a=None, b_x=None, lambda_=FAKE)
    p.update(over)
    return binding.Params(*(ctypes.c_void_p(v) if v is not None else None for v in p.values()))


def _prefill(d, p=None, x=FAKE, y=FAKE + 0x100, out=FAKE + 0x200, ws=FAKE, ws_bytes=1 << 20,
             state=None):
    lib = binding.load()
    p = p or _params()
    st = ctypes.byref(state) if state is not None else None
    return lib.rglru_block_prefill(ctypes.byref(d), ctypes.byref(p), ctypes.c_void_p(x) if x else None,
                                   ctypes.c_void_p(y) if y else None, None, st,
                                   ctypes.c_void_p(out) if out else None,
                                   ctypes.c_void_p(ws) if ws else None, ws_bytes, None)


@pytest.mark.parametrize("case,code", [
    (dict(batch=0), 1), (dict(seq_len=0), 1), (dict(heads=-1), 1), (dict(act_dtype=7), 1),
    (dict(head_dim=24), 2), (dict(head_dim=512), 2), (dict(gelu_tanh=2), 1),
])
def test_bad_dims_are_rejected(case, code):
    assert _prefill(_dims(**case)) == code


def test_bad_pointers_are_rejected():
    d = _dims()
    assert _prefill(d, x=None) == 1
    assert _prefill(d, x=FAKE + 2) == 1                      # misaligned activation
    assert _prefill(d, out=FAKE) == 1                          # out aliases x
    assert _prefill(d, p=_params(w_a=None)) == 1
    assert _prefill(d, p=_params(w_x=FAKE + 8)) == 1          # gate weights need 16 B
    assert _prefill(d, ws=None) == 3
    assert _prefill(d, ws_bytes=8) == 3
    assert _prefill(d, ws=FAKE + 16) == 1                     # workspace needs 256 B
    st = binding.State(ctypes.c_void_p(FAKE), None)
    assert _prefill(d, state=st) == 1
    d.c = 0.0
    assert _prefill(d) == 1


def test_decode_requires_state():
    lib = binding.load()
    d = _dims(seq_len=1)
    p = _params()
    rc = lib.rglru_block_decode(ctypes.byref(d), ctypes.byref(p), ctypes.c_void_p(FAKE),
                                ctypes.c_void_p(FAKE + 0x100), None, None,
                                ctypes.c_void_p(FAKE + 0x200), ctypes.c_void_p(FAKE), 1 << 20, None)
    assert rc == 1


def test_decode_steps_rejects_bad_arguments():
    lib = binding.load()
    d = _dims(seq_len=1)
    p = _params()
    st = binding.State(ctypes.c_void_p(FAKE + 0x1000), ctypes.c_void_p(FAKE + 0x2000))
    args = lambda steps, state, ws_bytes: (ctypes.byref(d), ctypes.byref(p), ctypes.c_void_p(FAKE),  # noqa: E731
                                           ctypes.c_void_p(FAKE + 0x100), None, steps, state,
                                           ctypes.c_void_p(FAKE + 0x200), ctypes.c_void_p(FAKE), ws_bytes, None)
    assert lib.rglru_block_decode_steps(*args(0, ctypes.byref(st), 1 << 20)) == 1      # no steps
    assert lib.rglru_block_decode_steps(*args(-3, ctypes.byref(st), 1 << 20)) == 1
    assert lib.rglru_block_decode_steps(*args(4, None, 1 << 20)) == 1                  # state required
    assert lib.rglru_block_decode_steps(*args(4, ctypes.byref(st), 8)) == 3            # workspace too small
    assert binding.decode_steps_workspace_size(d, 4) >= 16
    assert binding.decode_steps_workspace_size(d, 0) == 0
    k, n = ctypes.c_int(), ctypes.c_int()
    assert lib.rglru_decode_steps_plan(ctypes.byref(d), 0, ctypes.byref(k), ctypes.byref(n)) == 1


def test_mqa_rejects_bad_arguments():
    lib = binding.load()
    good = binding.make_mqa_dims(2, 64, 4, 256, 32)
    assert binding.mqa_workspace_size(good) >= 256 and binding.mqa_workspace_size(good, decode=True) >= 256
    for bad, code in ((binding.make_mqa_dims(2, 64, 4, 128, 32), 2),     # head_dim
                      (binding.make_mqa_dims(2, 64, 17, 256, 32), 2),    # too many query heads
                      (binding.make_mqa_dims(2, 64, 4, 256, 0), 1),      # window
                      (binding.make_mqa_dims(0, 64, 4, 256, 8), 1),      # batch
                      (binding.make_mqa_dims(2, 64, 4, 256, 32, scale=0.0), 1),    # score scale not > 0
                      (binding.make_mqa_dims(2, 64, 4, 256, 32, scale=-0.5), 1)):
        assert binding.mqa_workspace_size(bad) == 0
        rc = lib.rglru_mqa_prefill(ctypes.byref(bad), ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE + 0x100),
                                   ctypes.c_void_p(FAKE + 0x200), 0, ctypes.c_void_p(FAKE + 0x300), None,
                                   ctypes.c_void_p(FAKE), 1 << 30, None)
        assert rc == code
    rc = lib.rglru_mqa_decode(ctypes.byref(good), ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE + 0x100),
                              ctypes.c_void_p(FAKE + 0x200), None, ctypes.c_void_p(FAKE + 0x400),
                              ctypes.c_void_p(FAKE + 0x300), ctypes.c_void_p(FAKE), 1 << 30, None)
    assert rc == 1                                                       # positions required


def test_read_status_rejects_bad_workspace():
    lib = binding.load()
    assert lib.rglru_read_device_status(None, 256, None) == 1
    assert lib.rglru_read_device_status(ctypes.c_void_p(FAKE + 4), 256, None) == 1


def _backward(d, grads=None, x=FAKE, dout=FAKE + 0x300, ws=FAKE, ws_bytes=1 << 30):
    lib = binding.load()
    p = _params()
    if grads is None:
        grads = binding.Grads(*(ctypes.c_void_p(FAKE + 0x1000 * (i + 1)) for i in range(len(binding.GRAD_FIELDS))))
    g = ctypes.byref(grads) if grads is not False else None
    return lib.rglru_block_backward(ctypes.byref(d), ctypes.byref(p), ctypes.c_void_p(x) if x else None,
                                    ctypes.c_void_p(FAKE + 0x100), None, None,
                                    ctypes.c_void_p(dout) if dout else None, None, None, g,
                                    ctypes.c_void_p(ws) if ws else None, ws_bytes, None)


def test_backward_rejects_bad_arguments():
    d = _dims()
    assert binding.backward_workspace_size(d) > 4 * 2 * 16 * 128 * 4
    assert binding.backward_workspace_size(_dims(seq_len=0)) == 0
    assert binding.backward_plan(d) == (0, 4)
    assert _backward(_dims(head_dim=24)) == 2
    assert _backward(d, x=None) == 1
    assert _backward(d, dout=None) == 1
    assert _backward(d, dout=FAKE + 2) == 1                  # misaligned
    assert _backward(d, grads=False) == 1                     # no output struct
    fields = [ctypes.c_void_p(FAKE + 0x1000 * (i + 1)) for i in range(len(binding.GRAD_FIELDS))]
    fields[0] = None                                          # dx is required
    assert _backward(d, grads=binding.Grads(*fields)) == 1
    fields[0] = ctypes.c_void_p(FAKE)                         # dx aliases x
    assert _backward(d, grads=binding.Grads(*fields)) == 1
    assert _backward(d, ws=None) == 3
    assert _backward(d, ws_bytes=64) == 3
