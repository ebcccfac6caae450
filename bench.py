#!/usr/bin/env python
"""Benchmark of the RG-LRU recurrent block on B200: prefill tokens/s and HBM roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one full-sequence prefill (conv -> gates -> scan -> GeLU merge, state written back)
of the RecurrentGemma-2B-shaped workload: batch 8 x 2048 tokens, LRU width 2560 = 10 heads x
256, bf16 activations and gate weights, fp32 state; synthetic seeded inputs (no dataset, no
trained weights).  Inputs stay resident in HBM; one step moves 252 MB, more than the 126 MB L2,
so consecutive steps do not hit in L2.  The same JSON line also reports the single-token
decode workload (batch 256, width 2560, 1024 steps replayed from one CUDA graph).

N > 1 (torchrun): every rank runs its own replica of the workload on its own GPU (the block
shards over batch rows and heads with no exchange), the timed region is bracketed by a
barrier and a device synchronize on both sides, and the slowest rank's time is used.

--impl reference times the fp64 CPU oracle on the host cores on a bounded sample of the same
workload (rank 0 only).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_linear_recurrence_conv1d_b200 import inputs  # noqa: E402

WORKLOAD = "rg2b_bf16"
DECODE_WORKLOAD = "decode_bf16"
METRIC = "RG-LRU block prefill tokens/s (RecurrentGemma-2B-shaped, bf16, fp32 state)"

# DRAM bytes per launch measured by ncu (dram__bytes_read.sum + dram__bytes_write.sum) for a
# given kernel source; keyed by the sha256 of that source so a changed kernel reports null.
NCU_TRAFFIC = {
    # rg2b_bf16 step with state, one launch: 179.69 MB read + 88.97 MB written
    ("fused_prefill.cu", "e7f5915d5d3c3389"): 268657152,
}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def algorithmic_bytes(wl: inputs.Workload, tokens: int, with_state: bool = True) -> int:
    """x + y + out per token-channel, parameters once, state read + write once, reset mask."""
    es = 2 if wl.dtype == "bf16" else 4
    W, H, dh = wl.width, wl.heads, wl.head_dim
    b = 3 * es * tokens * W
    b += 2 * H * dh * dh * es + 4 * W * 4 + 4 * W * 4     # W_a, W_x, conv_w, conv_b/b_a/b_x/lambda
    if with_state:
        b += 2 * wl.batch * (4 * W + 3 * W * es)           # h and conv_tail, read + write
    if wl.doc_len is not None:
        b += tokens
    return b


def decode_bytes_per_step(wl: inputs.Workload) -> int:
    es = 2
    W = wl.width
    B = wl.batch
    return B * W * (3 * es + 2 * 4 + 2 * 3 * es)           # x, y, out; h r/w; tail r/w


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms while active."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return None
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": float(rows[0][2]),
                "samples": len(rows), "reasons": reasons,
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())}


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """The slowest rank's time: all-reduce MAX when a process group is up, else the value."""
    if dist is None or not dist.is_available() or not dist.is_initialized():
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, steps: int, ms: float) -> float:
    """Whole-job tokens/s: every rank processes its own replica (weak scaling)."""
    return tokens_per_rank * world * steps / (ms / 1000.0)


def env_rank():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def _sha(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


# ------------------------------------------------------------------ CPU oracle ------------

def oracle_prefill_rate(prob: inputs.Problem, target_s: float = 15.0, threads: int = 0):
    """Times the fp64 oracle on a bounded sample of the workload: whole rows with all their
    heads, the leading tokens of each, repeated until about target_s of CPU work has run.
    Returns (tokens/s, description, cores, seconds)."""
    import oracle
    wl = prob.wl
    cores = threads or len(os.sched_getaffinity(0))
    # calibrate: one row x 64 tokens (its heads run in parallel)
    t0 = time.perf_counter()
    oracle.prefill(prob.params, prob.x[:1, :64], prob.y[:1, :64], wl.heads, threads=cores)
    per_row_token = max((time.perf_counter() - t0) / 64, 1e-7)
    rows_per_wave = max(1, cores // wl.heads)
    tokens = int(min(wl.seq_len, max(64, target_s / per_row_token)))
    rows = min(wl.batch, rows_per_wave) if tokens == wl.seq_len else 1
    x, y = prob.x[:rows, :tokens], prob.y[:rows, :tokens]
    reset = None if prob.reset is None else prob.reset[:rows, :tokens]
    done, passes = 0, 0
    t0 = time.perf_counter()
    while True:
        oracle.prefill(prob.params, x, y, wl.heads, reset=reset, threads=cores)
        done += rows * tokens
        passes += 1
        if time.perf_counter() - t0 >= target_s:
            break
    dt = time.perf_counter() - t0
    desc = (f"{rows} row(s) x first {tokens} tokens x all {wl.heads} heads of {wl.name}, "
            f"{passes} pass(es)")
    return done / dt, desc, cores, dt


def oracle_backward_rate(prob: inputs.Problem, target_s: float = 3.0):
    """Times the fp64 oracle's backward (sequential, one core) on one row with all its heads,
    the leading tokens, sized to about target_s.  Returns (tokens/s, description, cores, s)."""
    import oracle
    wl = prob.wl
    rng = np.random.default_rng(1)

    def run(tokens):
        x, y = prob.x[:1, :tokens], prob.y[:1, :tokens]
        dout = inputs.make_activation(wl, rng, 1, tokens)
        reset = None if prob.reset is None else prob.reset[:1, :tokens]
        t0 = time.perf_counter()
        oracle.backward(prob.params, x, y, wl.heads, dout, reset=reset, gelu_tanh=wl.gelu_tanh)
        return time.perf_counter() - t0

    per_token = max(run(min(8, wl.seq_len)) / min(8, wl.seq_len), 1e-7)
    tokens = int(min(wl.seq_len, max(8, target_s / per_token)))
    dt = run(tokens)
    desc = f"1 row x first {tokens} tokens x all {wl.heads} heads of {wl.name}, one pass"
    return tokens / dt, desc, 1, dt


def run_reference(args):
    rank, world, _ = env_rank()
    if rank != 0:
        return
    wl = inputs.WORKLOADS[args.workload]
    prob = inputs.make_problem(wl, seed=0)
    vals = []
    desc, cores = "", 0
    for i in range(args.warmup + args.steps):
        rate, desc, cores, _ = oracle_prefill_rate(prob, target_s=args.ref_step_s)
        if i >= args.warmup:
            vals.append(rate)
    value = float(statistics.median(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * wl.batch * wl.seq_len / value, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "batch": wl.batch, "seq_len": wl.seq_len,
                   "heads": wl.heads, "head_dim": wl.head_dim, "width": wl.width},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU path --------------

def run_ours(args):
    import torch
    import torch.distributed as dist
    from gated_linear_recurrence_conv1d_b200 import binding

    rank, world, local = env_rank()
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", torch.cuda.current_device())
    lib = binding.load()
    del lib

    wl = inputs.WORKLOADS[args.workload]
    prob = inputs.make_problem(wl, seed=0)
    block = binding.RGLRUBlock(prob.params, wl.heads, wl.head_dim, wl.dtype, dev)
    x = binding.to_device(prob.x, dev)
    y = binding.to_device(prob.y, dev)
    reset = None if prob.reset is None else binding.to_device(prob.reset, dev)
    out = torch.empty_like(x)
    B, T, W = wl.batch, wl.seq_len, wl.width
    h = torch.zeros(B, W, device=dev)
    tail = torch.zeros(B, 3, W, device=dev, dtype=x.dtype)
    dims = block.dims(B, T)
    ws = binding.alloc_workspace(binding.prefill_workspace_size(dims), dev)
    stream = torch.cuda.current_stream()

    def step():
        binding.block_prefill(dims, block.params, x, y, out, ws, reset=reset, h=h, conv_tail=tail)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if binding.read_device_status(ws) != binding.RGLRU_OK:
        raise RuntimeError("device status not OK after warm-up")

    # ---- timed region: K prefill steps, per-launch CUDA events on the launching stream ----
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index if world == 1 else local) as clocks:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for i in range(args.steps):
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    total_ms = t_start.elapsed_time(t_end)
    launch_ms = [a.elapsed_time(b) for a, b in evs]
    status = binding.read_device_status(ws)
    if status != binding.RGLRU_OK:
        raise RuntimeError(f"device status {status} after the timed region")

    total_ms = max_over_ranks(total_ms, dist if world > 1 else None, dev)
    tokens_per_rank = B * T
    value = job_throughput(tokens_per_rank, world, args.steps, total_ms)

    # ---- roofline of the prefill kernel ----
    peak, peak_kind = measured_peaks()
    alg = algorithmic_bytes(wl, B * T, with_state=True)
    avg_launch_s = statistics.mean(launch_ms) / 1000.0
    achieved = alg / avg_launch_s / 1e9
    src = os.path.join(ROOT, "gated_linear_recurrence_conv1d_b200", "csrc", "fused_prefill.cu")
    if not os.path.exists(src):
        src = os.path.join(ROOT, "gated_linear_recurrence_conv1d_b200", "csrc", "generic.cu")
    traffic = NCU_TRAFFIC.get((os.path.basename(src), _sha(src)))

    # ---- end to end through the C ABI with pinned host buffers ----
    e2e_steps = max(3, min(args.steps, args.e2e_steps))
    e2e_ms = e2e_pipelined(binding, block, x, y, h, tail, reset, B, T, e2e_steps, dev, dist if world > 1 else None)
    e2e_value = job_throughput(tokens_per_rank, world, e2e_steps, e2e_ms)
    es = x.element_size()
    h2d = 2 * B * T * W * es
    d2h = B * T * W * es

    # ---- decode workload: 1024 single-token steps replayed from one CUDA graph ----
    decode = None
    if not args.no_decode:
        decode = bench_decode(args, dev)

    # ---- backward pass of the same prefill workload (portable kernels) ----
    backward = None
    if not args.no_backward:
        try:
            backward = bench_backward(args, dev)
        except Exception as exc:  # the prefill line above is the contract; report, do not lose it
            backward = {"error": f"{type(exc).__name__}: {exc}"}

    # ---- CPU oracle on a bounded sample (rank 0, N = 1 only) ----
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        rate, desc, cores, secs = oracle_prefill_rate(prob, target_s=args.cpu_seconds)
        cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": desc,
               "seconds": round(secs, 2)}
        # the same oracle on one core, on this workload and on the tiny fp32 one
        single = {}
        for name, pr in ((wl.name, prob),
                         ("tiny_f32", inputs.make_problem(inputs.WORKLOADS["tiny_f32"], seed=0))):
            r1, d1, _, s1 = oracle_prefill_rate(pr, target_s=min(3.0, args.cpu_seconds), threads=1)
            single[name] = {"value": r1, "unit": "tokens/s", "sample": d1, "seconds": round(s1, 2)}
        cpu["single_thread"] = single

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    clk = clocks.summary()
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": wl.name, "batch": B, "seq_len": T, "heads": wl.heads,
                   "head_dim": wl.head_dim, "width": W, "state": "fp32, read and written back",
                   "l2": "inputs larger than L2 (252 MB moved per step > 126 MB L2)",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_kind": peak_kind, "algorithmic_bytes_per_launch": alg,
                     "frac_of_8TBs": achieved / 8000.0, "kernel_source": os.path.basename(src)},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps * launches_per_prefill(dims),
        "clocks": clk,
        "decode": decode,
        "backward": backward,
    }
    print(json.dumps(line), flush=True)


def launches_per_prefill(dims) -> int:
    from gated_linear_recurrence_conv1d_b200 import binding
    return binding.prefill_launches(dims)


def e2e_pipelined(binding, block, x, y, h, tail, reset, B, T, steps, dev, dist=None, groups=4):
    """End-to-end time (ms) of `steps` prefill steps from pinned host buffers: every step copies
    x and y host -> device, runs the prefill through the C ABI and copies out device -> host.
    The batch is cut into row groups so that the copy engines (both directions) and the
    kernels overlap: group g's input copy, its prefill and its output copy run on three streams
    joined by events; device buffers alternate between two sets from one step to the next."""
    import torch
    if B % groups != 0:
        groups = 1
    R = B // groups
    x_h = x.cpu().pin_memory()
    y_h = y.cpu().pin_memory()
    out_h = torch.empty_like(x_h).pin_memory()
    xd = [x, torch.empty_like(x)]
    yd = [y, torch.empty_like(y)]
    od = [torch.empty_like(x), torch.empty_like(x)]
    s_in, s_cmp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
    dims = block.dims(R, T)
    ws = binding.alloc_workspace(binding.prefill_workspace_size(dims), dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_done = [[ev() for _ in range(groups)] for _ in range(2)]
    cmp_done = [[ev() for _ in range(groups)] for _ in range(2)]
    out_done = [[ev() for _ in range(groups)] for _ in range(2)]
    used = [[False] * groups for _ in range(2)]

    def one_step(i):
        b = i % 2
        for g in range(groups):
            rs = slice(g * R, (g + 1) * R)
            with torch.cuda.stream(s_in):
                if used[b][g]:
                    s_in.wait_event(cmp_done[b][g])      # the kernel of two steps ago has read them
                xd[b][rs].copy_(x_h[rs], non_blocking=True)
                yd[b][rs].copy_(y_h[rs], non_blocking=True)
                in_done[b][g].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(in_done[b][g])
                if used[b][g]:
                    s_cmp.wait_event(out_done[b][g])     # out of two steps ago has left
                binding.block_prefill(dims, block.params, xd[b][rs], yd[b][rs], od[b][rs], ws,
                                      reset=None if reset is None else reset[rs],
                                      h=h[rs], conv_tail=tail[rs], stream=s_cmp)
                cmp_done[b][g].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(cmp_done[b][g])
                out_h[rs].copy_(od[b][rs], non_blocking=True)
                out_done[b][g].record(s_out)
            used[b][g] = True

    for i in range(2):
        one_step(i)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    s_cmp.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(steps):
        one_step(i)
    s_in.wait_stream(s_out)
    e1.record(s_in)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    return max_over_ranks(ms, dist, dev)


def bench_decode(args, dev):
    import torch
    from gated_linear_recurrence_conv1d_b200 import binding

    wl = inputs.WORKLOADS[DECODE_WORKLOAD]
    if args.decode_steps > 0:
        wl = wl.scaled(decode_steps=args.decode_steps)
    steps = wl.decode_steps
    prob = inputs.make_problem(wl, seed=0)
    block = binding.RGLRUBlock(prob.params, wl.heads, wl.head_dim, wl.dtype, dev)
    xs = binding.to_device(prob.x, dev)      # [steps, B, W]
    ys = binding.to_device(prob.y, dev)
    outs = torch.empty_like(xs)
    h0 = binding.to_device(prob.h0, dev)
    t0 = binding.to_device(prob.tail0, dev)
    h = h0.clone()
    tail = t0.clone()
    dims = block.dims(wl.batch, 1)
    ws = binding.alloc_workspace(binding.decode_workspace_size(dims), dev)
    s = torch.cuda.Stream(device=dev)

    def run_all():
        for i in range(steps):
            binding.block_decode(dims, block.params, xs[i], ys[i], outs[i], h, tail, ws, stream=s)

    with torch.cuda.stream(s):
        run_all()                      # warm-up outside the graph
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        run_all()
    times = []
    for rep in range(4):
        h.copy_(h0)
        tail.copy_(t0)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(s):      # a graph replays on the current stream
            e0.record(s)
            g.replay()
            e1.record(s)
        torch.cuda.synchronize()
        if rep > 0:
            times.append(e0.elapsed_time(e1))
    ms = statistics.median(times)
    us_step = 1000.0 * ms / steps
    tok_s = wl.batch * steps / (ms / 1000.0)
    peak, _ = measured_peaks()
    bps = decode_bytes_per_step(wl)
    del g
    return {"workload": wl.name, "batch": wl.batch, "width": wl.width, "steps": steps,
            "value": tok_s, "unit": "tokens/s", "us_per_step": us_step,
            "effective_gbs": bps / (us_step * 1e-6) / 1e9,
            "effective_frac": bps / (us_step * 1e-6) / 1e9 / peak,
            "note": "state (h, conv_tail) and gate weights stay L2-resident across steps; "
                    "GB/s is algorithmic bytes over time (effective bandwidth)",
            "gpu_launches": steps * binding.decode_launches(dims)}


def bench_backward(args, dev, steps=3, warmup=1):
    """rglru_block_backward on the prefill workload (zero initial state, random dout)."""
    import torch
    from gated_linear_recurrence_conv1d_b200 import binding

    wl = inputs.WORKLOADS[args.workload]
    prob = inputs.make_problem(wl, seed=0)
    block = binding.RGLRUBlock(prob.params, wl.heads, wl.head_dim, wl.dtype, dev)
    x = binding.to_device(prob.x, dev)
    y = binding.to_device(prob.y, dev)
    rng = np.random.default_rng(1)
    dout = binding.to_device(inputs.make_activation(wl, rng, wl.batch, wl.seq_len), dev)
    B, T, W, H, dh = wl.batch, wl.seq_len, wl.width, wl.heads, wl.head_dim
    reset = None if prob.reset is None else binding.to_device(prob.reset, dev)
    dims = block.dims(B, T)
    ws = binding.alloc_workspace(binding.backward_workspace_size(dims), dev)
    shapes = {"dx": (B, T, W), "dy": (B, T, W), "dh0": (B, W), "dtail0": (B, 3, W),
              "dconv_w": (4, W), "dconv_b": (W,), "dw_a": (H, dh, dh), "dw_x": (H, dh, dh),
              "db_a": (W,), "db_x": (W,), "dlambda": (W,)}
    grads = {k: torch.empty(v, device=dev, dtype=torch.float32) for k, v in shapes.items()}
    s = torch.cuda.Stream(device=dev)
    for _ in range(warmup):
        binding.block_backward(dims, block.params, x, y, dout, grads, ws, reset=reset, stream=s)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(steps):
        binding.block_backward(dims, block.params, x, y, dout, grads, ws, reset=reset, stream=s)
    e1.record(s)
    torch.cuda.synchronize()
    if binding.read_device_status(ws) != binding.RGLRU_OK:
        raise RuntimeError("backward: device status not OK")
    ms = e0.elapsed_time(e1) / steps
    # algorithmic bytes: x, y, dout read (act dtype), dx, dy written (fp32), weights both ways
    es = x.element_size()
    alg = B * T * W * (3 * es + 8) + 2 * H * dh * dh * (es + 4)
    peak, _ = measured_peaks()
    line = {"workload": wl.name, "value": B * T / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms,
            "steps": steps, "kernels": "portable CUDA-core kernels, fp32 arithmetic",
            "effective_gbs": alg / (ms * 1e-3) / 1e9, "effective_frac": alg / (ms * 1e-3) / 1e9 / peak,
            "gpu_launches": steps * binding.backward_launches(dims)}
    if not args.no_cpu:
        rate, desc, cores, secs = oracle_backward_rate(prob, target_s=min(3.0, args.cpu_seconds))
        line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                "sample": desc, "seconds": round(secs, 2)}
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-step-s", type=float, default=4.0)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--decode-only", action="store_true",
                    help="time only the decode workload (prints its JSON object)")
    ap.add_argument("--decode-steps", type=int, default=0,
                    help="decode steps per graph replay (default: the workload's 1024)")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.decode_only:
        import torch
        dev = torch.device("cuda", torch.cuda.current_device())
        print(json.dumps(bench_decode(args, dev)))
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
