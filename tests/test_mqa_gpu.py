"""Local sliding-window MQA on the GPU (rglru_mqa_prefill / rglru_mqa_decode) against the fp64
oracle of oracle/mqa.py on the same bf16 inputs.

The kernels compute attention the usual tensor-core way: the rotated queries and keys and the
softmax weights P enter the MMAs as bf16 (relative rounding 2^-9 each), accumulation in fp32.
An output element O = sum_j P_j v_j then carries an error bounded by a small multiple of
sum_j P_j |v_j| (a rounding of P_j moves O by at most 2^-9 P_j |v_j|; a rounding of q or k
moves the score and so P_j relatively), not by a multiple of |O|, which cancellation can make
arbitrarily small.  The bar is therefore, element by element, |O - O_ref| <= 2^-6 sum_j P_j |v_j|
(the sum is the oracle's attention with |v| as the values; an emulation of these roundings in
fp64 stays below 2^-7 of it), next to the bf16 max-norm and RMS bars."""

import numpy as np
import pytest
import torch

from gated_linear_recurrence_conv1d_b200 import binding, inputs
from oracle import mqa
from tests.gpu_util import rel_err, rel_err_rms, to_np

pytestmark = pytest.mark.gpu

D = 256


def _bf16(rng, shape, s=1.0):
    return inputs.f32_to_bf16_bits((s * rng.standard_normal(shape)).astype(np.float32))


def _abs_bits(v):
    """|v| of bf16 bit patterns (the sign bit cleared: exact)."""
    return (v & 0x7FFF).astype(np.uint16)


def assert_attention_close(g, ref, pav, what):
    assert rel_err(g, ref) <= 2e-2, f"{what}: max-norm relative error {rel_err(g, ref):.3e}"
    assert rel_err_rms(g, ref) <= 5e-3, f"{what}: RMS relative error {rel_err_rms(g, ref):.3e}"
    ratio = np.max(np.abs(g.astype(np.float64) - ref) / np.maximum(pav, 1e-30))
    assert ratio <= 2.0 ** -6, f"{what}: |O - O_ref| / sum P|v| = {ratio:.3e} > 2^-6"


@pytest.mark.parametrize("B,T,H,w", [(1, 128, 1, 128), (2, 300, 3, 100), (1, 700, 10, 512), (2, 64, 2, 1)])
def test_mqa_prefill_matches_oracle(B, T, H, w):
    rng = np.random.default_rng(T + w)
    q, k, v = _bf16(rng, (B, T, H, D)), _bf16(rng, (B, T, D)), _bf16(rng, (B, T, D))
    dims = binding.make_mqa_dims(B, T, H, D, w)
    ws = binding.alloc_workspace(binding.mqa_workspace_size(dims))
    out = torch.empty(B, T, H, D, dtype=torch.bfloat16, device="cuda")
    td = lambda a: binding.to_device(a)  # noqa: E731
    binding.mqa_prefill(dims, td(q), td(k), td(v), out, ws, pos0=3)
    assert binding.read_device_status(ws) == binding.RGLRU_OK
    ref = mqa.prefill(q, k, v, window=w, pos0=3)
    pav = mqa.prefill(q, k, _abs_bits(v), window=w, pos0=3)
    assert_attention_close(to_np(out), ref, pav, f"mqa prefill B{B} T{T} H{H} w{w}")


@pytest.mark.parametrize("T0,H,w,steps", [
    (150, 4, 64, 40),      # a full ring that wraps many times
    (300, 10, 600, 6),     # a ring not yet full, window cut into splits (one of them empty)
    (700, 3, 600, 4),      # a full ring of several splits, the last one ragged
    (5, 16, 300, 3),       # a nearly empty ring (two empty splits), all 16 heads of the MMA's N
])
def test_mqa_decode_continues_the_prefill_through_the_ring(T0, H, w, steps):
    """Prefill T0 tokens with the cache, then decode steps; each step against the oracle's
    ring-buffer decode."""
    B = 2
    rng = np.random.default_rng(7)
    q, k, v = _bf16(rng, (B, T0, H, D)), _bf16(rng, (B, T0, D)), _bf16(rng, (B, T0, D))
    dims = binding.make_mqa_dims(B, T0, H, D, w)
    cache = torch.zeros(B, 2, w, D, dtype=torch.bfloat16, device="cuda")
    ws = binding.alloc_workspace(binding.mqa_workspace_size(dims))
    out = torch.empty(B, T0, H, D, dtype=torch.bfloat16, device="cuda")
    td = lambda a: binding.to_device(a)  # noqa: E731
    binding.mqa_prefill(dims, td(q), td(k), td(v), out, ws, pos0=0, cache=cache)
    rings = [mqa.RingCache(w, D) for _ in range(B)]
    arings = [mqa.RingCache(w, D) for _ in range(B)]        # the same keys, |v| as the values
    for b in range(B):
        for t in range(T0):
            kr = mqa.rope(mqa._f64(k[b, t]), np.array(t))
            rings[b].push(kr, mqa._f64(v[b, t]), t)
            arings[b].push(kr, np.abs(mqa._f64(v[b, t])), t)
    ddims = binding.make_mqa_dims(B, 1, H, D, w)
    wsd = binding.alloc_workspace(binding.mqa_workspace_size(ddims, decode=True))
    for s in range(steps):
        qd, kd, vd = _bf16(rng, (B, H, D)), _bf16(rng, (B, D)), _bf16(rng, (B, D))
        pos = np.array([T0 + s, T0 + s], dtype=np.int32)
        od = torch.empty(B, H, D, dtype=torch.bfloat16, device="cuda")
        binding.mqa_decode(ddims, td(qd), td(kd), td(vd), td(pos), cache, od, wsd)
        ref = np.stack([mqa.decode_step(rings[b], qd[b], kd[b], vd[b], int(pos[b])) for b in range(B)])
        pav = np.stack([mqa.decode_step(arings[b], qd[b], kd[b], _abs_bits(vd[b]), int(pos[b])) for b in range(B)])
        assert_attention_close(to_np(od), ref, pav, f"mqa decode step {s}")
    assert binding.read_device_status(wsd) == binding.RGLRU_OK


def test_mqa_decode_many_rows_multi_tile_parts():
    """Enough rows that the decode cuts each ring of 2048 into parts of several 128-slot tiles
    and a CTA streams several parts (running max / sum across tiles, queries of consecutive
    rows in flight together).  The ring is filled with random bf16 data, so slots past a short
    window hold values that must not leak; rows mix full rings (wrapped) and partial ones."""
    B, H, w = 80, 10, 2048
    rng = np.random.default_rng(11)
    cache_np = _bf16(rng, (B, 2, w, D))
    cache = binding.to_device(cache_np)
    pos = np.array([3000 + 37 * b if b % 4 else (b * 97) % 1900 for b in range(B)], dtype=np.int32)
    qd, kd, vd = _bf16(rng, (B, H, D)), _bf16(rng, (B, D)), _bf16(rng, (B, D))
    ddims = binding.make_mqa_dims(B, 1, H, D, w)
    wsd = binding.alloc_workspace(binding.mqa_workspace_size(ddims, decode=True))
    od = torch.empty(B, H, D, dtype=torch.bfloat16, device="cuda")
    td = lambda a: binding.to_device(a)  # noqa: E731
    binding.mqa_decode(ddims, td(qd), td(kd), td(vd), td(pos), cache, od, wsd)
    assert binding.read_device_status(wsd) == binding.RGLRU_OK
    got = to_np(od)
    kv = mqa._f64(cache_np)
    for b in range(B):
        ring, aring = mqa.RingCache(w, D), mqa.RingCache(w, D)
        ring.k[:], ring.v[:] = kv[b, 0], kv[b, 1]
        aring.k[:], aring.v[:] = kv[b, 0], np.abs(kv[b, 1])
        ring.filled = aring.filled = int(pos[b])
        ref = mqa.decode_step(ring, qd[b], kd[b], vd[b], int(pos[b]))
        pav = mqa.decode_step(aring, qd[b], kd[b], _abs_bits(vd[b]), int(pos[b]))
        assert_attention_close(got[b], ref, pav, f"mqa decode row {b} pos {pos[b]}")
