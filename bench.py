#!/usr/bin/env python
"""Benchmark of the RG-LRU recurrent block on B200: prefill / decode tokens/s and HBM roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one full-sequence prefill (conv -> gates -> scan -> GeLU merge, state read and
written back) through the C ABI.  The headline workload is the packed variable-length
prefill: batch 16 x 8192 tokens, LRU width 6144 = 24 heads x 256, documents of 64..4096
tokens packed per row with a segment-reset mask, bf16 activations and gate weights, fp32
state; synthetic seeded inputs (no dataset, no trained weights).  Inputs stay resident in HBM;
one step moves 4.8 GB, far more than the 126 MB L2.  The same JSON line carries one entry per
workload under "configs": the tiny fp32 check (L2 flushed between launches), the
RecurrentGemma-2B-shaped batch (B8 T2048, 10 x 256), the long-context row (B1 T65536,
16 x 256), the packed headline, and the single-token decode (batch 256, width 2560, 1024 steps
replayed from one CUDA graph); each with tokens/s, time per launch, algorithmic bytes, the
roofline fraction and the fp64 oracle timed on the host cores on a bounded sample.

N > 1 (torchrun): every rank runs its own replica of the workload on its own GPU (the block
shards over batch rows and heads with no exchange), the timed region is bracketed by a
barrier and a device synchronize on both sides, and the slowest rank's time is used.

--impl reference times the fp64 CPU oracle on the host cores on a bounded sample of the same
workload (rank 0 only).
"""

from __future__ import annotations

import argparse
import gc
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

WORKLOAD = "packed_bf16"                 # the headline: the largest single-GPU workload
PREFILL_WORKLOADS = ("tiny_f32", "rg2b_bf16", "long_bf16", "packed_bf16")
DECODE_WORKLOAD = "decode_bf16"
METRIC = "RG-LRU block tokens/s (prefill, decode) and achieved HBM GB/s"
# seconds of GPU time each non-headline prefill workload is timed for
CONFIG_SECONDS = 1.0

# DRAM bytes per launch measured by ncu (dram__bytes_read.sum + dram__bytes_write.sum) for a
# given kernel source; keyed by the sha256 of that source so a changed kernel reports null.
NCU_TRAFFIC = {
    # (kernel source, its sha256 prefix, workload): DRAM bytes read + written per launch, from one
    # ncu capture of that source (dram__bytes_read.sum and dram__bytes_write.sum on rg2b_bf16);
    # the packed workload's is that capture
    # scaled by the algorithmic bytes (every item moves the same tiles), the packed workload itself
    # being above the size a multi-pass capture may hold on the device
    ("fused_prefill.cu", "bf5e2316ce3e1637", "rg2b_bf16"): 236076288,
    ("fused_prefill.cu", "bf5e2316ce3e1637", "packed_bf16"): 4485236927,
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
    # each step a bounded sample, so that the whole run stays within about two minutes
    step_s = min(args.ref_step_s, 120.0 / (args.warmup + args.steps))
    for i in range(args.warmup + args.steps):
        rate, desc, cores, _ = oracle_prefill_rate(prob, target_s=step_s)
        if i >= args.warmup:
            vals.append(rate)
    value = float(statistics.median(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * wl.batch * wl.seq_len / value, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, world=1),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(wl: inputs.Workload, world: int) -> dict:
    moved = algorithmic_bytes(wl, wl.batch * wl.seq_len)
    cfg = {"workload": wl.name, "batch": wl.batch, "seq_len": wl.seq_len, "heads": wl.heads,
           "head_dim": wl.head_dim, "width": wl.width, "act_dtype": wl.dtype,
           "state": "fp32, read and written back",
           "parallelism": f"replicas x{world}"}
    if wl.doc_len is not None:
        cfg["documents"] = f"lengths U{{{wl.doc_len[0]}..{wl.doc_len[1]}}} packed per row, reset mask"
    cfg["l2"] = (f"inputs larger than L2 ({moved / 1e6:.0f} MB moved per step > 126 MB L2)"
                 if moved > 126e6 else "L2 flushed (256 MB write) between timed launches")
    return cfg


# ------------------------------------------------------------------ GPU path --------------

class PrefillRig:
    """One prefill workload resident on the device, run through the C ABI."""

    def __init__(self, binding, wl: inputs.Workload, dev):
        import torch
        self.binding, self.wl, self.dev = binding, wl, dev
        self.prob = inputs.make_problem(wl, seed=0)
        self.block = binding.RGLRUBlock(self.prob.params, wl.heads, wl.head_dim, wl.dtype, dev)
        self.x = binding.to_device(self.prob.x, dev)
        self.y = binding.to_device(self.prob.y, dev)
        self.reset = None if self.prob.reset is None else binding.to_device(self.prob.reset, dev)
        self.out = torch.empty_like(self.x)
        B, W = wl.batch, wl.width
        self.h = torch.zeros(B, W, device=dev)
        self.tail = torch.zeros(B, 3, W, device=dev, dtype=self.x.dtype)
        self.dims = self.block.dims(B, wl.seq_len)
        self.ws = binding.alloc_workspace(binding.prefill_workspace_size(self.dims), dev)

    def step(self, stream=None):
        self.binding.block_prefill(self.dims, self.block.params, self.x, self.y, self.out, self.ws,
                                   reset=self.reset, h=self.h, conv_tail=self.tail, stream=stream)

    def check_status(self, when: str):
        if self.binding.read_device_status(self.ws) != self.binding.RGLRU_OK:
            raise RuntimeError(f"{self.wl.name}: device status not OK {when}")


def time_prefill(rig: PrefillRig, steps: int, warmup: int, flush_l2: bool, dev, dist=None,
                 world: int = 1, clocks_gpu=None):
    """Times `steps` launches of the prefill on the current stream with CUDA events: per-launch
    events around each call and one pair around the whole loop (between barrier + synchronize
    on both sides).  With flush_l2 a 256 MB buffer is written between launches, outside the
    per-launch events.  Returns (total_ms, per-launch ms list, clock summary)."""
    import torch
    stream = torch.cuda.current_stream()
    flush = torch.empty(64 << 20, dtype=torch.float32, device=dev) if flush_l2 else None
    for _ in range(max(3, warmup)):
        rig.step()
    torch.cuda.synchronize()
    rig.check_status("after warm-up")
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(clocks_gpu if clocks_gpu is not None else dev.index) as clocks:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(steps):
            if flush is not None:
                flush.fill_(float(i))
            evs[i][0].record(stream)
            rig.step()
            evs[i][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    rig.check_status("after the timed region")
    per = [a.elapsed_time(b) for a, b in evs]
    total = sum(per) if flush_l2 else t0.elapsed_time(t1)
    return max_over_ranks(total, dist, dev), per, clocks.summary()


def prefill_entry(rig: PrefillRig, total_ms: float, per_ms, steps: int, world: int, clk) -> dict:
    wl = rig.wl
    B, T = wl.batch, wl.seq_len
    peak, peak_kind = measured_peaks()
    alg = algorithmic_bytes(wl, B * T, with_state=True)
    launch_ms = statistics.mean(per_ms)
    achieved = alg / (launch_ms / 1e3) / 1e9
    kernel, launches = rig.binding.prefill_plan(rig.dims)
    return {"workload": wl.name, "batch": B, "seq_len": T, "heads": wl.heads,
            "head_dim": wl.head_dim, "act_dtype": wl.dtype, "steps": steps,
            "value": job_throughput(B * T, world, steps, total_ms), "unit": "tokens/s",
            "ms_per_launch": launch_ms, "ms_per_launch_median": statistics.median(per_ms),
            "algorithmic_bytes_per_launch": alg, "achieved_gbs": achieved,
            "roofline_frac": achieved / peak, "peak_gbs": peak, "peak_kind": peak_kind,
            "frac_of_8TBs": achieved / 8000.0,
            "kernel": "tensor" if kernel == 1 else "generic", "launches_per_step": launches,
            "l2": workload_config(wl, world)["l2"], "clocks": clk}


def steps_for(ms_per_launch: float, seconds: float, lo: int = 5, hi: int = 2000) -> int:
    return int(min(hi, max(lo, seconds * 1000.0 / max(ms_per_launch, 1e-3))))


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
    binding.load()
    dd = dist if world > 1 else None
    clocks_gpu = dev.index if world == 1 else local
    cpu_on = rank == 0 and world == 1 and not args.no_cpu

    # ---- the headline workload: K timed steps ----
    head = PrefillRig(binding, inputs.WORKLOADS[args.workload], dev)
    wl = head.wl
    B, T, W = wl.batch, wl.seq_len, wl.width
    total_ms, per_ms, clk = time_prefill(head, args.steps, args.warmup, flush_l2=False, dev=dev,
                                         dist=dd, world=world, clocks_gpu=clocks_gpu)
    value = job_throughput(B * T, world, args.steps, total_ms)
    head_entry = prefill_entry(head, total_ms, per_ms, args.steps, world, clk)
    peak, peak_kind = measured_peaks()
    src = os.path.join(ROOT, "gated_linear_recurrence_conv1d_b200", "csrc", "fused_prefill.cu")
    traffic = NCU_TRAFFIC.get((os.path.basename(src), _sha(src), wl.name))
    roofline = {"bound": "hbm", "achieved": head_entry["achieved_gbs"], "peak": peak, "unit": "GB/s",
                "frac": head_entry["roofline_frac"], "traffic": traffic, "peak_kind": peak_kind,
                "algorithmic_bytes_per_launch": head_entry["algorithmic_bytes_per_launch"],
                "frac_of_8TBs": head_entry["frac_of_8TBs"], "kernel_source": os.path.basename(src),
                "workload": wl.name}

    # ---- end to end through the C ABI with pinned host buffers ----
    e2e_steps = max(3, min(args.steps, args.e2e_steps))
    e2e_ms = e2e_pipelined(binding, head.block, head.x, head.y, head.h, head.tail, head.reset, B, T,
                           e2e_steps, dev, dd)
    e2e_value = job_throughput(B * T, world, e2e_steps, e2e_ms)
    es = head.x.element_size()
    h2d = 2 * B * T * W * es + (0 if head.reset is None else B * T)
    d2h = B * T * W * es
    gpu_launches = args.steps * binding.prefill_launches(head.dims)

    cpu = None
    if cpu_on:
        rate, desc, cores, secs = oracle_prefill_rate(head.prob, target_s=args.cpu_seconds)
        cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": desc,
               "seconds": round(secs, 2)}
        head_entry["cpu_baseline"] = cpu
    configs = {wl.name: head_entry}
    del head
    gc.collect()
    torch.cuda.empty_cache()

    # ---- every other prefill workload, timed for about CONFIG_SECONDS each ----
    if not args.headline_only:
        for name in PREFILL_WORKLOADS:
            if name == wl.name:
                continue
            rig = PrefillRig(binding, inputs.WORKLOADS[name], dev)
            flush = algorithmic_bytes(rig.wl, rig.wl.batch * rig.wl.seq_len) <= 126e6
            # a short probe sizes the timed run (same launch configuration)
            _, probe, _ = time_prefill(rig, 3, 3, flush, dev, dd, world, clocks_gpu)
            n = steps_for(statistics.mean(probe), CONFIG_SECONDS)
            tot, per, ck = time_prefill(rig, n, 3, flush, dev, dd, world, clocks_gpu)
            entry = prefill_entry(rig, tot, per, n, world, ck)
            if cpu_on:
                r, d, c, sec = oracle_prefill_rate(rig.prob, target_s=args.config_cpu_seconds)
                entry["cpu_baseline"] = {"value": r, "unit": "tokens/s", "cores": c, "kind": "oracle",
                                         "sample": d, "seconds": round(sec, 2)}
            configs[name] = entry
            del rig
            gc.collect()
            torch.cuda.empty_cache()

    # ---- decode workload: 1024 single-token steps replayed from one CUDA graph ----
    if not args.no_decode:
        configs[DECODE_WORKLOAD] = bench_decode(args, dev, cpu_on)

    # ---- backward pass of the RecurrentGemma-2B-shaped prefill ----
    backward = None
    if not args.no_backward:
        try:
            backward = bench_backward(args, dev)
        except Exception as exc:  # the prefill line above is the contract; report, do not lose it
            backward = {"error": f"{type(exc).__name__}: {exc}"}

    extras = {}
    if not args.no_extras:
        for name, fn in (("layer", bench_layer), ("mqa", bench_mqa)):
            try:
                extras[name] = fn(args, dev)
            except Exception as exc:  # the headline line is the contract; report, do not lose it
                extras[name] = {"error": f"{type(exc).__name__}: {exc}"}
            gc.collect()
            torch.cuda.empty_cache()

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    cfg = workload_config(wl, world)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": cfg, "roofline": roofline, "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": gpu_launches, "clocks": clk, "configs": configs, "backward": backward,
        "layer": extras.get("layer"), "mqa": extras.get("mqa"),
    }
    print(json.dumps(line), flush=True)


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


def oracle_decode_rate(prob: inputs.Problem, target_s: float = 3.0):
    """Times the fp64 oracle's decode on the host cores: successive single-token steps of the
    decode workload from its initial state, for about target_s.  Returns (tokens/s, description,
    cores, seconds)."""
    import oracle
    wl = prob.wl
    cores = len(os.sched_getaffinity(0))
    h = prob.h0.astype(np.float64).copy()
    tail = oracle.tail_from_act(prob.tail0).copy()
    done = 0
    t0 = time.perf_counter()
    while done < wl.decode_steps:
        oracle.decode(prob.params, prob.x[done], prob.y[done], wl.heads, h, tail, threads=cores)
        done += 1
        if time.perf_counter() - t0 >= target_s:
            break
    dt = time.perf_counter() - t0
    desc = f"first {done} of {wl.decode_steps} steps x batch {wl.batch} x all {wl.heads} heads of {wl.name}"
    return wl.batch * done / dt, desc, cores, dt


def bench_decode(args, dev, cpu_on: bool = False):
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
    single = {"value": tok_s, "unit": "tokens/s", "us_per_step": us_step,
              "effective_gbs": bps / (us_step * 1e-6) / 1e9,
              "effective_frac": bps / (us_step * 1e-6) / 1e9 / peak,
              "note": "one rglru_block_decode launch per step, 1024 steps replayed from one CUDA "
                      "graph; state (h, conv_tail) and gate weights stay L2-resident across steps; "
                      "GB/s is algorithmic bytes (26 B per row-channel per step) over time",
              "gpu_launches": steps * binding.decode_launches(dims)}

    # the same steps in one persistent launch (rglru_block_decode_steps): the state stays on chip
    wss = binding.alloc_workspace(binding.decode_steps_workspace_size(dims, steps), dev)
    ptimes = []
    for rep in range(4):
        h.copy_(h0)
        tail.copy_(t0)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s)
        binding.block_decode_steps(dims, block.params, xs, ys, outs, h, tail, wss, stream=s)
        e1.record(s)
        torch.cuda.synchronize()
        if rep > 0:
            ptimes.append(e0.elapsed_time(e1))
    if binding.read_device_status(wss) != binding.RGLRU_OK:
        raise RuntimeError("persistent decode: device status not OK")
    pms = statistics.median(ptimes)
    pus = 1000.0 * pms / steps
    W = wl.width
    # algorithmic bytes of the whole launch: x, y, out per step; the state read and written
    # once; gate weights and parameters once
    p_alg = steps * wl.batch * W * 6 + wl.batch * W * (8 + 12) + 2 * wl.heads * 256 * 256 * 2 + 8 * W * 4
    p_gbs = p_alg / (pms * 1e-3) / 1e9
    kind, launches = binding.decode_steps_plan(dims, steps)
    entry = {"workload": wl.name, "batch": wl.batch, "width": wl.width, "steps": steps,
             "value": wl.batch * steps / (pms / 1000.0), "unit": "tokens/s", "us_per_step": pus,
             "path": "rglru_block_decode_steps: all steps in one persistent launch",
             "algorithmic_bytes_per_launch": p_alg, "achieved_gbs": p_gbs, "roofline_frac": p_gbs / peak,
             "peak_gbs": peak, "kernel": "tensor" if kind == 1 else "generic",
             "gpu_launches": launches, "single_step": single}
    if cpu_on:
        r, d, c, sec = oracle_decode_rate(prob, target_s=min(3.0, args.config_cpu_seconds))
        entry["cpu_baseline"] = {"value": r, "unit": "tokens/s", "cores": c, "kind": "oracle", "sample": d,
                                 "seconds": round(sec, 2)}
    return entry


def bench_backward(args, dev, steps=3, warmup=1):
    """rglru_block_backward on the prefill workload (zero initial state, random dout)."""
    import torch
    from gated_linear_recurrence_conv1d_b200 import binding

    wl = inputs.WORKLOADS["rg2b_bf16"]
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
            "steps": steps,
            "kernels": "tensor-core path" if binding.backward_plan(dims)[0] == 1 else "portable kernels",
            "effective_gbs": alg / (ms * 1e-3) / 1e9, "effective_frac": alg / (ms * 1e-3) / 1e9 / peak,
            "gpu_launches": steps * binding.backward_launches(dims)}
    if not args.no_cpu:
        rate, desc, cores, secs = oracle_backward_rate(prob, target_s=min(3.0, args.cpu_seconds))
        line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                "sample": desc, "seconds": round(secs, 2)}
    return line


def bench_layer(args, dev, steps=10):
    """rglru_layer_forward on the RecurrentGemma-2B-shaped batch with model width 2560: the three
    projections (tensor-core GEMMs) around the block, against the same computation with torch
    matmuls (cuBLAS) around rglru_block_prefill."""
    import torch
    from gated_linear_recurrence_conv1d_b200 import binding

    wl = inputs.WORKLOADS["rg2b_bf16"]
    D = 2560
    prob = inputs.make_problem(wl, seed=0)
    rng = np.random.default_rng(2)
    B, T, W = wl.batch, wl.seq_len, wl.width
    block = binding.RGLRUBlock(prob.params, wl.heads, wl.head_dim, wl.dtype, dev)
    u = torch.randn(B, T, D, device=dev).to(torch.bfloat16)
    wx = (torch.randn(D, W, device=dev) / D ** 0.5).to(torch.bfloat16)
    wy = (torch.randn(D, W, device=dev) / D ** 0.5).to(torch.bfloat16)
    wo = (torch.randn(W, D, device=dev) / W ** 0.5).to(torch.bfloat16)
    del rng
    pj = binding.make_projections(D, wx, wy, wo)
    dims = block.dims(B, T)
    ws = binding.alloc_workspace(binding.layer_workspace_size(dims), dev)
    out = torch.empty(B, T, D, dtype=torch.bfloat16, device=dev)
    h = torch.zeros(B, W, device=dev)
    tail = torch.zeros(B, 3, W, dtype=torch.bfloat16, device=dev)

    def ours():
        binding.layer_forward(dims, block.params, pj, u, out, ws, h=h, conv_tail=tail)

    wsb = binding.alloc_workspace(binding.prefill_workspace_size(dims), dev)
    z = torch.empty(B, T, W, dtype=torch.bfloat16, device=dev)

    def composed():
        x = torch.matmul(u, wx)
        y = torch.matmul(u, wy)
        binding.block_prefill(dims, block.params, x, y, z, wsb, h=h, conv_tail=tail)
        torch.matmul(z, wo)

    def timeit(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    ms = timeit(ours)
    if binding.read_device_status(ws) != binding.RGLRU_OK:
        raise RuntimeError("layer: device status not OK")
    ms_c = timeit(composed)
    flops = 2.0 * B * T * D * W * 3
    return {"workload": "rg2b_bf16 with model width 2560", "batch": B, "seq_len": T, "model_dim": D,
            "value": B * T / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms,
            "projection_tflops": flops / (ms * 1e-3) / 1e12,
            "torch_matmuls_around_block": {"value": B * T / (ms_c * 1e-3), "unit": "tokens/s", "ms_per_step": ms_c},
            "gpu_launches": steps * binding.layer_plan(dims, pj)[1]}


def bench_mqa(args, dev, steps=10, dsteps=32):
    """Local sliding-window MQA, RecurrentGemma-2B-shaped: 10 query heads x 256 over one key /
    value head, window 2048; prefill of batch 8 x 2048 tokens and decode of batch 256 against
    full rings."""
    import torch
    from gated_linear_recurrence_conv1d_b200 import binding

    B, T, H, d, w = 8, 2048, 10, 256, 2048
    q = torch.randn(B, T, H, d, device=dev).to(torch.bfloat16)
    k = torch.randn(B, T, d, device=dev).to(torch.bfloat16)
    v = torch.randn(B, T, d, device=dev).to(torch.bfloat16)
    out = torch.empty_like(q)
    dims = binding.make_mqa_dims(B, T, H, d, w)
    ws = binding.alloc_workspace(binding.mqa_workspace_size(dims), dev)
    for _ in range(3):
        binding.mqa_prefill(dims, q, k, v, out, ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        binding.mqa_prefill(dims, q, k, v, out, ws)
    e1.record()
    torch.cuda.synchronize()
    if binding.read_device_status(ws) != binding.RGLRU_OK:
        raise RuntimeError("mqa prefill: device status not OK")
    ms = e0.elapsed_time(e1) / steps
    # score and weighted-sum flops over the causal window (every query sees min(t + 1, w) keys)
    keys = sum(min(t + 1, w) for t in range(T))
    flops = 4.0 * B * H * d * keys
    peak_tf = measured_tensor_peak()
    pre = {"workload": f"B{B} T{T} {H} query heads x {d}, window {w}", "value": B * T / (ms * 1e-3),
           "unit": "tokens/s", "ms_per_step": ms, "tflops": flops / (ms * 1e-3) / 1e12,
           "tensor_frac": flops / (ms * 1e-3) / 1e12 / peak_tf, "tensor_peak_tflops": peak_tf}
    Bd = 256
    cache = torch.randn(Bd, 2, w, d, device=dev).to(torch.bfloat16)
    ddims = binding.make_mqa_dims(Bd, 1, H, d, w)
    wsd = binding.alloc_workspace(binding.mqa_workspace_size(ddims, decode=True), dev)
    qd = torch.randn(dsteps, Bd, H, d, device=dev).to(torch.bfloat16)
    kd = torch.randn(dsteps, Bd, d, device=dev).to(torch.bfloat16)
    vd = torch.randn(dsteps, Bd, d, device=dev).to(torch.bfloat16)
    od = torch.empty(Bd, H, d, dtype=torch.bfloat16, device=dev)
    pos = [torch.full((Bd,), 4096 + s, dtype=torch.int32, device=dev) for s in range(dsteps)]
    for s in range(3):
        binding.mqa_decode(ddims, qd[s], kd[s], vd[s], pos[s], cache, od, wsd)
    torch.cuda.synchronize()
    e0.record()
    for s in range(dsteps):
        binding.mqa_decode(ddims, qd[s], kd[s], vd[s], pos[s], cache, od, wsd)
    e1.record()
    torch.cuda.synchronize()
    if binding.read_device_status(wsd) != binding.RGLRU_OK:
        raise RuntimeError("mqa decode: device status not OK")
    us = 1000.0 * e0.elapsed_time(e1) / dsteps
    bytes_step = Bd * 2 * w * d * 2 + Bd * (H + 2) * d * 2 * 2
    peak, _ = measured_peaks()
    dec = {"workload": f"B{Bd} {H} query heads x {d}, full rings of {w}", "value": Bd / (us * 1e-6),
           "unit": "tokens/s", "us_per_step": us, "achieved_gbs": bytes_step / (us * 1e-6) / 1e9,
           "roofline_frac": bytes_step / (us * 1e-6) / 1e9 / peak}
    return {"prefill": pre, "decode": dec}


def measured_tensor_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"])
    except Exception:
        return 1590.0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="oracle seconds on the headline workload")
    ap.add_argument("--config-cpu-seconds", type=float, default=4.0,
                    help="oracle seconds on each other workload")
    ap.add_argument("--ref-step-s", type=float, default=4.0)
    ap.add_argument("--headline-only", action="store_true",
                    help="time only the headline workload (no per-workload entries)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--decode-only", action="store_true",
                    help="time only the decode workload (prints its JSON object)")
    ap.add_argument("--decode-steps", type=int, default=0,
                    help="decode steps per graph replay (default: the workload's 1024)")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the layer and MQA entries")
    ap.add_argument("--extras-only", action="store_true",
                    help="time only the backward, layer and MQA entries (prints their JSON object)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.decode_only:
        import torch
        dev = torch.device("cuda", torch.cuda.current_device())
        print(json.dumps(bench_decode(args, dev)))
    elif args.extras_only:
        import torch
        dev = torch.device("cuda", torch.cuda.current_device())
        out = {} if args.no_backward else {"backward": bench_backward(args, dev)}
        out["layer"] = bench_layer(args, dev)
        out["mqa"] = bench_mqa(args, dev)
        print(json.dumps(out))
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
