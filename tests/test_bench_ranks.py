"""Host-side logic of the multi-process bench, on CPU with the gloo backend (world size 2):
the timed region uses the slowest rank, the value counts every rank's replica, and only rank 0
runs the CPU reference arm."""

import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local_ms = [12.5, 20.0][rank]
    ms = bench.max_over_ranks(local_ms, dist, "cpu")
    value = bench.job_throughput(16384, world, 10, ms)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, ms, value))


def test_max_over_ranks_and_weak_scaling_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, value in res:
        assert ms == 20.0                                   # the slowest rank's time
        assert value == pytest.approx(16384 * 2 * 10 / 0.020)


def test_single_process_paths():
    assert bench.max_over_ranks(3.0) == 3.0
    assert bench.job_throughput(100, 1, 2, 1000.0) == pytest.approx(200.0)


def test_reference_arm_runs_on_rank0_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        workload = "tiny_f32"
        steps = 1
        warmup = 0
        gpus = 2
        ref_step_s = 0.1

    bench.run_reference(Args())
    assert capsys.readouterr().out == ""


def test_oracle_backward_rate_on_a_small_sample():
    """The CPU baseline beside the backward measurement: a bounded oracle sample."""
    from gated_linear_recurrence_conv1d_b200 import inputs
    wl = inputs.WORKLOADS["tiny_f32"].scaled(seq_len=40)
    prob = inputs.make_problem(wl, seed=0)
    rate, desc, cores, secs = bench.oracle_backward_rate(prob, target_s=0.05)
    assert rate > 0 and cores == 1 and secs > 0
    assert "tiny_f32" in desc
