"""Rows of one chunk (T <= 32), repeated in fresh processes: the tensor-core prefill's two CTAs of
a head both read the old conv history of every row in its first chunk while each writes the new
history of its own half at the row's last chunk -- here the same chunk.  The kernel reads a copy
of the history taken before the launch, so the outcome must not depend on which CTA runs first.
Each fresh process (a new context, new scheduling) runs several seeds and shapes and requires
the exact conv history and the parity bar every time."""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_CHILD = r"""
import numpy as np
import oracle
from gated_linear_recurrence_conv1d_b200 import binding, inputs
from tests.gpu_util import GpuProblem, assert_close, to_np
base = inputs.WORKLOADS["rg2b_bf16"]
for T in (1, 2, 3, 5, 17, 32):
    for seed in range(3):
        wl = base.scaled(batch=3, seq_len=T, heads=2, random_state=True)
        prob = inputs.make_problem(wl, seed=100 * T + seed)
        gp = GpuProblem(prob)
        out, h, tail, status = gp.prefill(use_state=True)
        assert status == binding.RGLRU_OK, status
        r_out, r_h, r_tail = oracle.prefill(prob.params, prob.x, prob.y, wl.heads, reset=prob.reset,
                                            h0=prob.h0, tail0=prob.tail0)
        np.testing.assert_array_equal(to_np(tail), r_tail)
        assert_close(to_np(out), r_out, "bf16", f"T{T} seed{seed} out")
        assert_close(to_np(h), r_h, "bf16", f"T{T} seed{seed} h")
print("ok")
"""


@pytest.mark.parametrize("run", range(3))
def test_one_chunk_rows_in_fresh_processes(run):
    env = dict(os.environ, PYTHONPATH=ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""))
    r = subprocess.run([sys.executable, "-c", _CHILD], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), (r.stdout[-2000:], r.stderr[-4000:])
