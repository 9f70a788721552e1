#!/usr/bin/env python
"""Benchmark: causal self-attention forward + backward TFLOP/s on B200.

One step = gptattn_fwd + gptattn_bwd (all kernels of the path) over one batch of
the workload, through the C ABI.  Default workload: the GPT-2 124M attention
shape (B=16, T=1024, 12 heads of 64, bf16), seeded synthetic inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload gpt2_124m]

FLOPs are counted causally (half of dense): fwd 2*B*nh*T^2*hs, bwd 2.5x that.
The L2 is flushed (256 MiB write) before every timed step, outside the step's
CUDA events.  Under torchrun every rank runs its own batch (weak scaling, no
collective on the data path); the step time is the max over ranks.

Prints one JSON line (rank 0).  --impl reference times the fp64 CPU oracle on
a bounded sample of the same workload instead (test infrastructure, the only
place besides the cpu_baseline leg where bench.py runs it).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="gpt2_124m")
    p.add_argument("--cpu-sample-seconds", type=float, default=12.0)
    p.add_argument("--skip-cpu-baseline", action="store_true")
    p.add_argument("--profile-run", action="store_true",
                   help="warm-up and timed steps only (no clock sampling, e2e or CPU leg): for ncu captures")
    p.add_argument("--dropout-run", action="store_true",
                   help="warm-up and timed fwd+bwd steps with attention dropout p = 0.1 only: for ncu captures")
    p.add_argument("--block-run", action="store_true",
                   help="only the attention sub-block call, warm-up + steps times: for ncu captures of its kernels")
    return p.parse_args()


# DRAM traffic per launch of the dominant kernel, from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum) of the same workload; reported
# only while the sources it was taken on are unchanged (sha256 over the files).
MEASURED_TRAFFIC = {
    ("bwd_bf16_sm100", "gpt2_124m"): {
        "bytes": 198.058752e6 + 82.057728e6,
        "sources": ("bwd_h64_sm100.cu", "sm100_ptx.cuh", "kernels.h"),
        "sha256": "3b2c15c069969d607dc060d5b80adc03d35e1174593cbfc9f4850780b2cfccac",
        "capture": "profiles/bwd_h64_persistent_gpt2_124m.md",
    },
}


def measured_traffic(kernel: str, workload: str):
    import hashlib
    rec = MEASURED_TRAFFIC.get((kernel, workload))
    if rec is None:
        return None
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "causal_self_attention_gptattn_b200", "csrc")
    try:
        for f in rec["sources"]:
            with open(os.path.join(csrc, f), "rb") as fh:
                h.update(fh.read())
    except OSError:
        return None
    return rec["bytes"] if h.hexdigest() == rec["sha256"] else None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return FALLBACK_PEAKS, "fallback"


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while work runs."""

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={CLOCK_FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.gpu_index)],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i in range(4) if r[i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------------------- CPU oracle timing
def time_oracle(w, budget_s: float, seed: int = 0):
    """Time the fp64 oracle on whole (batch, head) pairs of the workload until
    about budget_s seconds have elapsed.  Returns (TFLOP/s, cores, sample text)."""
    import numpy as np

    import oracle
    from causal_self_attention_gptattn_b200.workloads import workload_inputs

    qkv, dy = workload_inputs(w, B=1)
    q = qkv.double().numpy()
    g = dy.double().numpy()
    C, hs, nh = w.C, w.hs, w.n_head
    heads_done = 0
    elapsed = 0.0
    while elapsed < budget_s and heads_done < w.B * nh:
        h = heads_done % nh
        cols = np.r_[h * hs:(h + 1) * hs, C + h * hs:C + (h + 1) * hs, 2 * C + h * hs:2 * C + (h + 1) * hs]
        qh = np.ascontiguousarray(q[:, :, cols])
        gh = np.ascontiguousarray(g[:, :, h * hs:(h + 1) * hs])
        t0 = time.perf_counter()
        oracle.forward(qh, 1)
        oracle.backward(qh, gh, 1)
        elapsed += time.perf_counter() - t0
        heads_done += 1
    flops = 3.5 * 2.0 * heads_done * w.T * w.T * w.hs
    sample = (f"{heads_done} (batch, head) pairs of {w.name} (T={w.T}, hs={w.hs}), fwd+bwd each, "
              f"fp64 oracle; {elapsed:.1f} s")
    return flops / elapsed / 1e12, oracle.num_threads(), sample, elapsed


def run_reference(args, w, rank):
    if rank != 0:
        return
    import oracle
    cores = oracle.num_threads()
    # size each step so the whole run stays within a few minutes
    per_pair = None
    steps_run = 0
    total_s = 0.0
    total_flops = 0.0
    budget_total = 150.0
    start = time.perf_counter()
    for k in range(args.warmup + args.steps):
        if time.perf_counter() - start > budget_total and k > args.warmup:
            break
        per_step_budget = budget_total / (args.warmup + args.steps)
        v, _, sample, el = time_oracle(w, per_step_budget)
        if k >= args.warmup:
            steps_run += 1
            total_s += el
            total_flops += v * 1e12 * el
    value = total_flops / total_s / 1e12 if total_s > 0 else 0.0
    # each timed "step" is a bounded sample of the workload's (batch, head) pairs; ms_per_step is
    # the time a whole step (all B * n_head pairs) takes at the sampled rate
    full_step_flops = 3.5 * 2.0 * w.B * w.n_head * w.T * w.T * w.hs
    line = {
        "impl": "reference", "metric": "causal attention fwd+bwd TFLOP/s (bf16, 1 B200)", "value": value,
        "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": steps_run, "warmup": args.warmup,
        "ms_per_step": 1e3 * full_step_flops / (value * 1e12) if value > 0 else None,
        "ms_per_sample": 1e3 * total_s / max(steps_run, 1), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {**w.describe(), "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"per step: {sample}"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- GPU arm
def make_block_call(ga, w, dev, s):
    """Device buffers of the pre-LN attention sub-block at the workload's B, T, C (seeded
    inputs) and a closure that enqueues one gptattn_attn_block_fwd call on stream s."""
    import torch

    from causal_self_attention_gptattn_b200.workloads import block_inputs
    B, T, C, nh = w.B, w.T, w.C, w.n_head
    xb_c, pb_c = block_inputs(B, T, C, seed=2000 + w.index)
    bufs = {"x": xb_c.to(dev), **{k: v.to(dev) for k, v in pb_c.items()},
            "qkv": torch.empty(B, T, 3 * C, dtype=torch.bfloat16, device=dev),
            "y": torch.empty(B, T, C, dtype=torch.bfloat16, device=dev),
            "lse": torch.empty(B, nh, T, dtype=torch.float32, device=dev),
            "out": torch.empty(B, T, C, dtype=torch.bfloat16, device=dev)}

    def call():
        b = bufs
        ga.check(ga.gptattn_attn_block_fwd(b["x"], b["ln_w"], b["ln_b"], b["w_attn"], b["b_attn"], b["w_proj"],
                                           b["b_proj"], b["qkv"], b["y"], b["lse"], b["out"], B, T, C, nh,
                                           ga.GPTATTN_BF16, s), "gptattn_attn_block_fwd")
    return call, bufs


# --------------------------------------------------------------------------- ranks
# One process per GPU under torchrun.  Each rank runs the unchanged single-GPU op on a batch
# of its own (independent problems: weak scaling, no collective on the data path); the only
# collectives are the barriers around the timed region and the max of the ranks' times.
def rank_seed(w, rank: int) -> int:
    """Seed of a rank's synthetic batch: every rank draws different inputs."""
    return 1000 + w.index + 7919 * rank


def init_ranks(world: int, backend: str = "nccl", device=None):
    """Process group for world > 1 (NCCL on GPUs; the CPU tests use gloo), short timeout; None at world 1."""
    if world <= 1:
        return None
    import datetime

    import torch.distributed as dist
    kw = {"device_id": device} if backend == "nccl" and device is not None else {}
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return dist


def max_over_ranks(dist, x: float, device="cpu") -> float:
    """The largest of the ranks' values (the job's time is the slowest rank's)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(world: int, steps: int, flops_per_step: float, max_total_ms: float) -> float:
    """Whole-job throughput: every rank ran `steps` steps of `flops_per_step` FLOPs, and the job
    took as long as its slowest rank."""
    return world * steps * flops_per_step / (max_total_ms / 1e3) / 1e12


def time_other_workload(ga, name, dev, s, flush, steps):
    """One fwd+bwd step of another workload timed like the headline one (L2 flushed before
    each step, CUDA events around it), then a per-kernel pass; returns its record."""
    import torch

    from causal_self_attention_gptattn_b200.workloads import by_name, workload_inputs
    ow = by_name(name)
    B, T, C, nh = ow.B, ow.T, ow.C, ow.n_head
    dt = ga.GPTATTN_BF16
    qkv_c, dy_c = workload_inputs(ow)
    qkv, dy = qkv_c.to(dev), dy_c.to(dev)
    y = torch.empty(B, T, C, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, nh, T, dtype=torch.float32, device=dev)
    dqkv = torch.empty_like(qkv)
    nb = ga.gptattn_bwd_workspace_bytes(B, T, C, nh, dt)
    ws = torch.empty(nb, dtype=torch.uint8, device=dev)

    def step():
        ga.check(ga.gptattn_fwd(qkv, y, lse, B, T, C, nh, dt, s), "gptattn_fwd")
        ga.check(ga.gptattn_bwd(qkv, y, lse, dy, dqkv, ws, nb, B, T, C, nh, dt, s), "gptattn_bwd")

    for _ in range(5):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    Ko = max(1, min(steps, 200))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(Ko)]
    for a, b_ in evs:
        flush.zero_()
        a.record(s)
        step()
        b_.record(s)
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b_) for a, b_ in evs) / Ko
    ga.gptattn_profile_enable(4 * Ko + 64)
    for _ in range(Ko):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    per = {}
    for kname, kms in ga.gptattn_profile_read(4 * Ko + 64):
        per.setdefault(kname, []).append(kms)
    ga.gptattn_profile_enable(0)
    ga.check(ga.gptattn_get_device_status(s), f"device status after {name}")
    kern = {k: statistics.mean(v) for k, v in per.items()}
    peaks, src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    bwd_ms = kern.get("bwd_bf16_sm100")
    fwd_ms = kern.get("fwd_bf16_sm100")
    return {"config": ow.describe(), "steps": Ko, "ms_per_step": ms, "flops_per_step": ow.flops_fwd_bwd(),
            "value": ow.flops_fwd_bwd() / (ms / 1e3) / 1e12, "unit": "TFLOP/s",
            "pct_of_measured_bf16_burst": ow.flops_fwd_bwd() / (ms / 1e3) / 1e12 / peak,
            "kernels_ms": kern,
            "roofline": {"bound": "tensor", "kernel": "bwd_bf16_sm100",
                         "achieved": (ow.flops_bwd() / (bwd_ms / 1e3) / 1e12 if bwd_ms else None), "peak": peak,
                         "unit": "TFLOP/s",
                         "frac": (ow.flops_bwd() / (bwd_ms / 1e3) / 1e12 / peak if bwd_ms else None),
                         "peak_source": f"{src} bf16 burst"},
            "fwd_frac_of_peak": (ow.flops_fwd() / (fwd_ms / 1e3) / 1e12 / peak if fwd_ms else None),
            "l2": "flushed before every timed step"}


def run_ours(args, w, rank, world, local_rank):
    import torch

    from causal_self_attention_gptattn_b200 import gptattn as ga
    from causal_self_attention_gptattn_b200.workloads import make_inputs

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = init_ranks(world, "nccl", dev)

    dt = ga.GPTATTN_BF16 if w.dtype == "bf16" else ga.GPTATTN_F32
    B, T, C, nh = w.B, w.T, w.C, w.n_head
    qkv_c, dy_c = make_inputs(B, T, nh, w.hs, dtype=w.torch_dtype, seed=rank_seed(w, rank), recipe=w.recipe,
                              qkv_scale=w.qkv_scale)
    qkv = qkv_c.to(dev)
    dy = dy_c.to(dev)
    y = torch.empty(B, T, C, dtype=w.torch_dtype, device=dev)
    lse = torch.empty(B, nh, T, dtype=torch.float32, device=dev)
    dqkv = torch.empty_like(qkv)
    nbytes = ga.gptattn_bwd_workspace_bytes(B, T, C, nh, dt)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)  # 256 MiB > 126 MB L2
    s = torch.cuda.current_stream(dev)
    if args.block_run:
        block_call, _ = make_block_call(ga, w, dev, s)
        for _ in range(args.warmup + args.steps):
            flush.zero_()
            block_call()
        torch.cuda.synchronize()
        ga.check(ga.gptattn_get_device_status(s), "device status after the sub-block calls")
        if dist is not None:
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps({"block_run": "ok", "calls": args.warmup + args.steps}), flush=True)
        return

    if args.dropout_run:
        o = ga.Options(dropout_p=0.1, dropout_seed=1234)
        nb_o = ga.gptattn_bwd_opts_workspace_bytes(B, T, C, nh, o, dt)
        ws_o = torch.empty(max(nb_o, 256), dtype=torch.uint8, device=dev)
        for _ in range(args.warmup + args.steps):
            flush.zero_()
            ga.check(ga.gptattn_fwd_opts(qkv, y, lse, B, T, C, nh, o, dt, s), "gptattn_fwd_opts")
            ga.check(ga.gptattn_bwd_opts(qkv, y, lse, dy, dqkv, ws_o, nb_o, B, T, C, nh, o, dt, s), "gptattn_bwd_opts")
        torch.cuda.synchronize()
        ga.check(ga.gptattn_get_device_status(s), "device status after the dropout steps")
        if dist is not None:
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps({"dropout_run": "ok", "steps": args.warmup + args.steps}), flush=True)
        return

    def step(q=qkv, g=dy):
        ga.check(ga.gptattn_fwd(q, y, lse, B, T, C, nh, dt, s), "gptattn_fwd")
        ga.check(ga.gptattn_bwd(q, y, lse, g, dqkv, ws, nbytes, B, T, C, nh, dt, s), "gptattn_bwd")

    def barrier():
        if dist is not None:
            dist.barrier()

    def slowest(x: float) -> float:
        return max_over_ranks(dist, x, dev)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    ga.check(ga.gptattn_get_device_status(s), "device status after warm-up")

    K = args.steps
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    sampler = ClockSampler(local_rank)
    if not args.profile_run:
        sampler.start()
        time.sleep(0.25)
    launches0 = ga.gptattn_launch_count()
    barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    for k in range(K):
        flush.zero_()
        starts[k].record(s)
        step()
        ends[k].record(s)
    torch.cuda.synchronize()
    barrier()
    wall1 = time.perf_counter()
    launches = ga.gptattn_launch_count() - launches0
    # keep the same loop running (untimed) so the clock sampler sees >= ~1.5 s of load
    extra_until = wall0 + (0.0 if args.profile_run else 1.5)
    while time.perf_counter() < extra_until:
        for _ in range(50):
            flush.zero_()
            step()
        torch.cuda.synchronize()
    clocks = sampler.stop()
    ga.check(ga.gptattn_get_device_status(s), "device status after timing")

    # The same steps back to back with no flush in between (the L2 keeps what the previous
    # step left, as in a training loop that repeats one layer's shapes): reported alongside.
    hot = None
    if not args.profile_run:
        Kh = max(1, min(K, 500))
        h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        h0.record(s)
        for _ in range(Kh):
            step()
        h1.record(s)
        torch.cuda.synchronize()
        hot_ms = slowest(h0.elapsed_time(h1))
        hot = {"steps": Kh, "ms_per_step": hot_ms / Kh, "value": aggregate_tflops(world, Kh, w.flops_fwd_bwd(), hot_ms),
               "unit": "TFLOP/s", "l2": "not flushed between steps"}

    # Second timed pass, same steps, with the library recording a pair of CUDA events
    # around each kernel on the launching stream: per-kernel durations for the roofline.
    # (Kept out of the headline pass: an event between two kernels stops the next one
    # from starting its CTAs while the previous one drains.)
    Kp = max(1, min(K, 200))
    ga.gptattn_profile_enable(4 * Kp + 64)
    torch.cuda.synchronize()
    for _ in range(Kp):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    prof = ga.gptattn_profile_read(4 * Kp + 64)
    ga.gptattn_profile_enable(0)

    step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    total_ms = slowest(sum(step_ms))
    flops = w.flops_fwd_bwd()
    value = aggregate_tflops(world, K, flops, total_ms)

    # per-kernel durations recorded by the library inside the timed loop
    per_kernel = {}
    for name, ms in prof:
        per_kernel.setdefault(name, []).append(ms)
    kern_avg = {k: statistics.mean(v) for k, v in per_kernel.items()}

    # ---- end to end through the C ABI with host buffers (copies inside the timed region)
    # Every step copies its inputs host->device from pinned memory and its outputs (y and
    # dqkv) device->host, as a user streaming batches would: copies in on one stream,
    # compute on another, copies out on a third, device buffers double-buffered, so that
    # step k's compute overlaps step k+1's input copy and step k-1's output copy.
    qkv_h = qkv_c.pin_memory()
    dy_h = dy_c.pin_memory()
    y_h = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    dqkv_h = torch.empty(dqkv.shape, dtype=dqkv.dtype).pin_memory()
    bufs = [{"qkv": torch.empty_like(qkv), "dy": torch.empty_like(dy), "y": torch.empty_like(y),
             "lse": torch.empty_like(lse), "dqkv": torch.empty_like(dqkv)} for _ in range(2)]
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)

    def step_into(bf):
        ga.check(ga.gptattn_fwd(bf["qkv"], bf["y"], bf["lse"], B, T, C, nh, dt, s), "gptattn_fwd")
        ga.check(ga.gptattn_bwd(bf["qkv"], bf["y"], bf["lse"], bf["dy"], bf["dqkv"], ws, nbytes, B, T, C, nh, dt, s),
                 "gptattn_bwd")

    def e2e_run(n_steps, t0=None, t1=None):
        ev = lambda: torch.cuda.Event()
        h2d_done = [ev() for _ in range(n_steps)]
        comp_done = [ev() for _ in range(n_steps)]
        d2h_done = [ev() for _ in range(n_steps)]
        if t0 is not None:
            t0.record(s_in)
        for k in range(n_steps):
            bf = bufs[k & 1]
            if k >= 2:
                s_in.wait_event(comp_done[k - 2])  # step k-2 no longer reads these inputs
            with torch.cuda.stream(s_in):
                bf["qkv"].copy_(qkv_h, non_blocking=True)
                bf["dy"].copy_(dy_h, non_blocking=True)
            h2d_done[k].record(s_in)
            s.wait_event(h2d_done[k])
            if k >= 2:
                s.wait_event(d2h_done[k - 2])  # step k-2's outputs have been copied out
            flush.zero_()
            step_into(bf)
            comp_done[k].record(s)
            s_out.wait_event(comp_done[k])
            with torch.cuda.stream(s_out):
                y_h.copy_(bf["y"], non_blocking=True)
                dqkv_h.copy_(bf["dqkv"], non_blocking=True)
            d2h_done[k].record(s_out)
        if t1 is not None:
            s_out.wait_event(d2h_done[n_steps - 1])
            t1.record(s_out)
        torch.cuda.synchronize()

    Ke = 0 if args.profile_run else max(1, min(K, 200))
    e2e_run(3)
    barrier()
    e2e_ms = 0.0
    if Ke:
        e_start = torch.cuda.Event(enable_timing=True)
        e_end = torch.cuda.Event(enable_timing=True)
        e2e_run(Ke, e_start, e_end)
        e2e_ms = e_start.elapsed_time(e_end)
    barrier()
    e2e_ms = slowest(e2e_ms)
    e2e_value = aggregate_tflops(world, Ke, flops, e2e_ms) if Ke else None
    h2d = qkv_h.numel() * qkv_h.element_size() + dy_h.numel() * dy_h.element_size()
    d2h = y_h.numel() * y_h.element_size() + dqkv_h.numel() * dqkv_h.element_size()

    # ---- local window (gptattn_fwd_window + gptattn_bwd_window), 256-token band: the same step
    # with only the band's key tiles; FLOPs counted over the visible (query, key) pairs,
    # 14 * hs per pair (4 fwd + 10 bwd), which is the causal count 7*B*nh*T^2*hs for a full band.
    banded = None
    if not args.profile_run:
        W = 256
        pairs = sum(min(t + 1, W) for t in range(T))
        flops_w = 14.0 * w.hs * B * nh * pairs

        def step_w():
            ga.check(ga.gptattn_fwd_window(qkv, y, lse, B, T, C, nh, W, dt, s), "gptattn_fwd_window")
            ga.check(ga.gptattn_bwd_window(qkv, y, lse, dy, dqkv, ws, nbytes, B, T, C, nh, W, dt, s),
                     "gptattn_bwd_window")

        for _ in range(5):
            flush.zero_()
            step_w()
        torch.cuda.synchronize()
        Kw = max(1, min(K, 200))
        tw = 0.0
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(Kw)]
        for a, b_ in evs:
            flush.zero_()
            a.record(s)
            step_w()
            b_.record(s)
        torch.cuda.synchronize()
        tw = sum(a.elapsed_time(b_) for a, b_ in evs)
        ga.check(ga.gptattn_get_device_status(s), "device status after the banded steps")
        banded = {"window": W, "steps": Kw, "ms_per_step": tw / Kw, "flops_per_step": flops_w,
                  "value": flops_w * Kw / (tw / 1e3) / 1e12, "unit": "TFLOP/s",
                  "flop_count": "14*hs per visible (query, key) pair, exact band",
                  "pct_of_measured_bf16_burst": flops_w * Kw / (tw / 1e3) / 1e12 /
                  float(load_peaks()[0].get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))}

    # ---- deterministic backward (gptattn_bwd_det): the same step with dQ partials stored per
    # (query tile, key tile) and summed in a fixed order instead of reduce-added.
    det = None
    if not args.profile_run:
        nb_det = ga.gptattn_bwd_det_workspace_bytes(B, T, C, nh, dt)
        ws_det = torch.empty(max(nb_det, 256), dtype=torch.uint8, device=dev)

        def step_det():
            ga.check(ga.gptattn_fwd(qkv, y, lse, B, T, C, nh, dt, s), "gptattn_fwd")
            ga.check(ga.gptattn_bwd_det(qkv, y, lse, dy, dqkv, ws_det, nb_det, B, T, C, nh, 1 << 30, dt, s),
                     "gptattn_bwd_det")

        for _ in range(5):
            flush.zero_()
            step_det()
        torch.cuda.synchronize()
        Kd = max(1, min(K, 200))
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(Kd)]
        for a, b_ in evs:
            flush.zero_()
            a.record(s)
            step_det()
            b_.record(s)
        torch.cuda.synchronize()
        td = sum(a.elapsed_time(b_) for a, b_ in evs)
        ga.check(ga.gptattn_get_device_status(s), "device status after the deterministic steps")
        det = {"steps": Kd, "ms_per_step": td / Kd, "value": flops * Kd / (td / 1e3) / 1e12, "unit": "TFLOP/s",
               "workspace_bytes": nb_det}
        del ws_det

    # ---- attention dropout p = 0.1 (gptattn_fwd_opts + gptattn_bwd_opts): the same step with
    # the Philox keep mask generated in the forward and again in the backward; FLOPs counted as
    # for the plain step (the mask adds no matrix work).
    drop = None
    if not args.profile_run:
        o = ga.Options(dropout_p=0.1, dropout_seed=1234)
        nb_o = ga.gptattn_bwd_opts_workspace_bytes(B, T, C, nh, o, dt)

        def step_drop():
            ga.check(ga.gptattn_fwd_opts(qkv, y, lse, B, T, C, nh, o, dt, s), "gptattn_fwd_opts")
            ga.check(ga.gptattn_bwd_opts(qkv, y, lse, dy, dqkv, ws, nb_o, B, T, C, nh, o, dt, s), "gptattn_bwd_opts")

        for _ in range(5):
            flush.zero_()
            step_drop()
        torch.cuda.synchronize()
        Ko = max(1, min(K, 200))
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(Ko)]
        for a, b_ in evs:
            flush.zero_()
            a.record(s)
            step_drop()
            b_.record(s)
        torch.cuda.synchronize()
        to = sum(a.elapsed_time(b_) for a, b_ in evs)
        ga.gptattn_profile_enable(4 * Ko + 64)
        for _ in range(Ko):
            flush.zero_()
            step_drop()
        torch.cuda.synchronize()
        per_d = {}
        for kname, kms in ga.gptattn_profile_read(4 * Ko + 64):
            per_d.setdefault(kname, []).append(kms)
        ga.gptattn_profile_enable(0)
        ga.check(ga.gptattn_get_device_status(s), "device status after the dropout steps")
        drop = {"dropout_p": 0.1, "steps": Ko, "ms_per_step": to / Ko, "value": flops * Ko / (to / 1e3) / 1e12,
                "unit": "TFLOP/s", "flop_count": "as the plain step",
                "kernels_ms": {k: statistics.mean(v) for k, v in per_d.items()}}

    # ---- decode (gptattn_decode): the last position of every sequence over the same qkv as a
    # key/value cache; HBM-bound, so its roofline is the measured copy bandwidth.  L2 flushed
    # before every call.  Also a large cache (B=64, T=4096 at this head layout) for the
    # asymptotic bandwidth.
    decode = None
    if not args.profile_run:
        peaks_d, src_d = load_peaks()
        hbm = float(peaks_d.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        yd = torch.empty(B, C, dtype=w.torch_dtype, device=dev)
        ld = torch.empty(B, nh, dtype=torch.float32, device=dev)

        def time_decode(q, Bq, Tq, reps, flush_each):
            for _ in range(3):
                ga.check(ga.gptattn_decode(q, yd if Bq == B else yl, ld if Bq == B else ll, Bq, Tq, Tq, C, nh, dt, s),
                         "gptattn_decode")
            torch.cuda.synchronize()
            tot = 0.0
            for _ in range(reps):
                if flush_each:
                    flush.zero_()
                a = torch.cuda.Event(enable_timing=True)
                b_ = torch.cuda.Event(enable_timing=True)
                a.record(s)
                ga.check(ga.gptattn_decode(q, yd if Bq == B else yl, ld if Bq == B else ll, Bq, Tq, Tq, C, nh, dt, s),
                         "gptattn_decode")
                b_.record(s)
                torch.cuda.synchronize()
                tot += a.elapsed_time(b_)
            return tot / reps

        ms_d = time_decode(qkv, B, T, 50, True)
        kv_bytes = B * T * 2 * C * qkv.element_size()
        BL, TL = 64, 4096
        ql = torch.empty(BL, TL, 3 * C, dtype=w.torch_dtype, device=dev).normal_()
        yl = torch.empty(BL, C, dtype=w.torch_dtype, device=dev)
        ll = torch.empty(BL, nh, dtype=torch.float32, device=dev)
        ms_l = time_decode(ql, BL, TL, 20, False)
        kv_l = BL * TL * 2 * C * ql.element_size()
        del ql
        decode = {"workload": f"{w.name}: last position of each of the B={B} sequences over T={T} cached keys",
                  "us_per_call": ms_d * 1e3, "kv_bytes": kv_bytes, "achieved_gbs": kv_bytes / ms_d / 1e6,
                  "frac_of_hbm": kv_bytes / ms_d / 1e6 / hbm, "peak_source": f"{src_d} copy bandwidth",
                  "large_cache": {"B": BL, "T": TL, "us_per_call": ms_l * 1e3, "kv_bytes": kv_l,
                                  "achieved_gbs": kv_l / ms_l / 1e6, "frac_of_hbm": kv_l / ms_l / 1e6 / hbm}}

    # ---- the attention sub-block (gptattn_attn_block_fwd): LayerNorm -> c_attn -> causal
    # attention -> c_proj + residual at this workload's B, T, C; bf16 only.  Whole-call time
    # with CUDA events (L2 flushed before each call), then per-kernel times from the library's
    # event records (launch order: layernorm, c_attn GEMM, attention forward, c_proj GEMM).
    attn_block = None
    if not args.profile_run and dt == ga.GPTATTN_BF16:
        peaks_b, src_b = load_peaks()
        tc_peak = float(peaks_b.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        hbm_b = float(peaks_b.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        block_call, block_bufs = make_block_call(ga, w, dev, s)

        for _ in range(5):
            flush.zero_()
            block_call()
        torch.cuda.synchronize()
        Kb = max(1, min(K, 100))
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(Kb)]
        for a, b_ in evs:
            flush.zero_()
            a.record(s)
            block_call()
            b_.record(s)
        torch.cuda.synchronize()
        ms_b = sum(a.elapsed_time(b_) for a, b_ in evs) / Kb
        ga.gptattn_profile_enable(4 * Kb + 16)
        for _ in range(Kb):
            flush.zero_()
            block_call()
        torch.cuda.synchronize()
        recs = ga.gptattn_profile_read(4 * Kb + 16)
        ga.gptattn_profile_enable(0)
        ga.check(ga.gptattn_get_device_status(s), "device status after the sub-block calls")
        parts = {"layernorm": [], "c_attn": [], "attention": [], "c_proj": []}
        for i in range(0, len(recs) - 3, 4):
            for key, (_, ms) in zip(parts, recs[i:i + 4]):
                parts[key].append(ms)
        pm = {k: (statistics.mean(v) if v else None) for k, v in parts.items()}
        M = B * T
        fl = {"c_attn": 2.0 * M * C * 3 * C, "attention": w.flops_fwd(), "c_proj": 2.0 * M * C * C}
        ln_bytes = 2 * M * C * 2 + 4 * C
        attn_block = {
            "workload": f"{w.name}: pre-LN attention sub-block forward, x [{B},{T},{C}] bf16",
            "ms_per_call": ms_b, "flops_per_call": sum(fl.values()),
            "value": sum(fl.values()) / (ms_b / 1e3) / 1e12, "unit": "TFLOP/s",
            "kernels_ms": pm,
            "gemm_tflops": {k: (fl[k] / (pm[k] / 1e3) / 1e12 if pm[k] else None) for k in ("c_attn", "c_proj")},
            "gemm_frac_of_bf16_peak": {k: (fl[k] / (pm[k] / 1e3) / 1e12 / tc_peak if pm[k] else None)
                                       for k in ("c_attn", "c_proj")},
            "layernorm_gbs": (ln_bytes / (pm["layernorm"] / 1e3) / 1e9 if pm["layernorm"] else None),
            "layernorm_frac_of_hbm": (ln_bytes / (pm["layernorm"] / 1e3) / 1e9 / hbm_b if pm["layernorm"] else None),
            "peak_source": f"{src_b} bf16 burst / copy bandwidth", "calls": Kb}
        del block_bufs

    # ---- the other bf16 workloads of the configuration list, each timed like the headline
    # workload (L2 flushed before every step, CUDA events per step), plus per-kernel times
    # and the main backward kernel's fraction of the bf16 peak.  Single GPU only.
    others = None
    if not args.profile_run and world == 1 and dt == ga.GPTATTN_BF16:
        others = {}
        for oname in ("baby_gpt", "gpt2_124m", "gpt2_1p5b", "long_context"):
            if oname != w.name:
                others[oname] = time_other_workload(ga, oname, dev, s, flush, K)

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks, peak_src = load_peaks()
    dominant = "bwd_bf16_sm100" if dt == ga.GPTATTN_BF16 else "bwd_dkv_f32"
    dom_ms = kern_avg.get(dominant)
    dom_flops = w.flops_bwd()  # the main backward kernel does all 5 backward matmuls
    roofline = None
    if dom_ms:
        achieved = dom_flops / (dom_ms / 1e3) / 1e12
        peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        roofline = {"bound": "tensor", "kernel": dominant, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "peak_source": f"{peak_src} bf16 burst",
                    "traffic": measured_traffic(dominant, args.workload), "traffic_unit": "bytes per launch",
                    "avg_ms": dom_ms}

    cpu = None
    if world == 1 and not (args.skip_cpu_baseline or args.profile_run):
        v, cores, sample, _ = time_oracle(w, args.cpu_sample_seconds)
        cpu = {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample}

    line = {
        "metric": "causal attention fwd+bwd TFLOP/s (bf16, 1 B200)",
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": total_ms / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic",
        "config": {**w.describe(), "parallelism": f"dp{world} (independent batches per GPU)",
                   "flops_per_step_per_gpu": flops,
                   "l2": "flushed before every timed step (256 MiB write, outside the step events)"},
        "pct_of_peak": {"measured_bf16_burst": value / world / float(peaks.get("bf16_tflops", 1590.0)),
                        "datasheet_2250": value / world / 2250.0},
        "kernels_ms": kern_avg,
        "hot_l2": hot,
        "value_exact_triangle": value * (T + 1) / T,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": Ke, "ms_per_step": (e2e_ms / Ke if Ke else None),
                "overlap": "copies in / compute / copies out on three streams, device buffers double-buffered"},
        "gpu_launches": launches,
        "decode": decode,
        "attn_block": attn_block,
        "window": banded,
        "deterministic": det,
        "dropout": drop,
        "other_workloads": others,
        "clocks": clocks,
        "wall_s_timed": wall1 - wall0,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    from causal_self_attention_gptattn_b200.workloads import by_name
    w = by_name(args.workload)
    if args.impl == "reference":
        run_reference(args, w, rank)
        return
    run_ours(args, w, rank, world, local_rank)


if __name__ == "__main__":
    main()
