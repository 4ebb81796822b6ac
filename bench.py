#!/usr/bin/env python
"""Benchmark of the H3 transport hot path on B200: effective HBM GB/s.

One step is one pass of the whole path on the ragged 32k-token workload
(T = 32768 packed tokens, W = 6 virtual ranks, heads 10,10,9,9,9,9, 8 packed
segments):

  1. h3_partition            token/head ranges, segments clipped and rebased (host)
  2. h3_seq_to_head          packed QKV [32768, 3, 56, 128] -> 6 x [32768, 3, H_j, 128]
  3. h3_head_to_seq          back to [32768, 3, 56, 128], chunked one plane per
                             launch under the 896,000,000-byte window
  4. h3_ragged_reduce_scatter 6 BF16 partials [32768, 7168] + bias -> 6 x [T_r, 7168]

value = algorithmic bytes of all steps (each input read once + each output
written once) / device time, summed over GPUs.  Every kernel's inputs are
1.4-2.8 GB, far larger than the 126 MB L2, so no flush is needed between
steps.  With --gpus N (torchrun) every GPU runs an independent replica of the
step: the path has no exchange between GPUs when all virtual ranks share one
GPU's memory.

--impl reference times the plain CPU oracle (oracle/) on the host cores on a
bounded sample of the same workload; it is the slow reference, not a target.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "relayout + reduce-scatter effective HBM GB/s and % of B200 HBM peak"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # nominal B200 HBM3e bandwidth, for a second percentage only
STEP_T, STEP_W, STEP_P, STEP_SEGS, STEP_SEED = 32768, 6, 3, 8, 2
WINDOW = 896_000_000


# ---------------------------------------------------------------------------
# host-side helpers (no GPU needed; covered by the gloo tests)
# ---------------------------------------------------------------------------

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(x: float, device) -> float:
    """Largest value of x over all ranks (x itself without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device) -> float:
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def throughput_gbs(bytes_per_step_per_gpu: float, steps: int, n_gpus: int, seconds: float) -> float:
    """Whole-job GB/s: every GPU's bytes over the slowest GPU's time."""
    return bytes_per_step_per_gpu * steps * n_gpus / seconds / 1e9


def load_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# The sources each measured kernel is compiled from.
KERNEL_SOURCES = {
    "seq_to_head": ("relayout.cu", "device_access.cuh", "bulk_copy.cuh", "h3rr_internal.h"),
    "head_to_seq": ("relayout.cu", "device_access.cuh", "bulk_copy.cuh", "h3rr_internal.h"),
    "ragged_reduce_scatter": ("reduce_scatter.cu", "bf16_sum.cuh", "device_access.cuh", "h3rr_internal.h"),
}


def kernel_source_digest(kernel: str) -> str:
    """Digest of the sources `kernel` is compiled from: traffic figures taken
    with other sources are not reported."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "ragged_reduce_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernels changed since it was taken."""
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
            table = json.load(f)
    except (OSError, ValueError):
        return None
    entry = table.get(kernel)
    if not entry or kernel not in KERNEL_SOURCES or entry.get("source_digest") != kernel_source_digest(kernel):
        return None
    return entry.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines: list[str] = []

    def __enter__(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "100"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self) -> dict:
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# the step on the GPU
# ---------------------------------------------------------------------------

class Step:
    """Device buffers and calls of one step of the path (inputs resident)."""

    def __init__(self, device, T=STEP_T, W=STEP_W, P=STEP_P, n_segs=STEP_SEGS, seed=STEP_SEED,
                 relayout=True, reduce=True):
        import ragged_reduce_b200 as rr
        self.rr = rr
        self.device = device
        self.T, self.W, self.P, self.H, self.D = T, W, P, wl.H3_HEADS, wl.H3_HEAD_DIM
        self.C = wl.H3_HIDDEN
        self.bounds = wl.segment_bounds(T, n_segs, seed)
        self.part = rr.partition(T, self.H, W, self.bounds)
        if relayout:
            self.qkv = wl.normal_bf16((T, P, self.H, self.D), seed, 1.0, device)
            self.send = rr.split_rows(self.qkv, self.part.token_starts)
            self.heads = rr.alloc_head_side(T, P, self.H, self.D, W, device)
            self.back_full, self.back = rr.alloc_seq_side(T, P, self.H, self.D, W, device)
        if reduce:
            rw = wl.ReduceWorkload("step", T=T, C=self.C, W=W, seed=seed + 100)
            self.partials, self.bias = wl.partials_and_bias(rw, device)
            self.partial_list = list(self.partials.unbind(0))
            self.red_full, self.red_out = rr.alloc_reduce_outputs(T, self.C, W, device)
        relayout_bytes = T * P * self.H * self.D * 2 * 2
        reduce_bytes = (W + 1) * T * self.C * 2 + self.C * 2
        self.kernel_bytes = {"seq_to_head": relayout_bytes, "head_to_seq": relayout_bytes,
                             "ragged_reduce_scatter": reduce_bytes}
        self.bytes_per_step = sum(self.kernel_bytes.values())
        self.launches = {}

    def run(self, events=None, stream=None):
        rr = self.rr
        if events is not None:
            events[0].record(stream)
        rr.partition(self.T, self.H, self.W, self.bounds)
        i1 = rr.seq_to_head(self.send, self.heads, stream=stream)
        if events is not None:
            events[1].record(stream)
        i2 = rr.head_to_seq(self.heads, self.back, window_bytes=WINDOW, stream=stream)
        if events is not None:
            events[2].record(stream)
        i3 = rr.ragged_reduce_scatter(self.partial_list, self.bias, self.red_out, stream=stream)
        if events is not None:
            events[3].record(stream)
        self.launches = {"seq_to_head": i1["launches"], "head_to_seq": i2["launches"],
                         "ragged_reduce_scatter": i3["launches"]}
        return i1["launches"] + i2["launches"] + i3["launches"]

    def verify(self) -> bool:
        """Round trip and reduce spot check (not timed)."""
        ok = torch.equal(self.back_full.view(torch.int16), self.qkv.view(torch.int16))
        acc = self.partials[0].float()
        for k in range(1, self.W):
            acc += self.partials[k].float()
        acc += self.bias.float()
        ok = ok and torch.equal(self.red_full.view(torch.int16), acc.to(torch.bfloat16).view(torch.int16))
        return bool(ok)

    def host_io(self):
        """Pinned host copies of the step's inputs and room for its results."""
        return {
            "qkv": self.qkv.cpu().pin_memory(),
            "partials": self.partials.cpu().pin_memory(),
            "bias": self.bias.cpu().pin_memory(),
            "back": torch.empty(self.back_full.shape, dtype=torch.bfloat16).pin_memory(),
            "red": torch.empty(self.red_full.shape, dtype=torch.bfloat16).pin_memory(),
        }

    @staticmethod
    def io_bytes(io):
        h2d = sum(io[k].numel() * 2 for k in ("qkv", "partials", "bias"))
        d2h = sum(io[k].numel() * 2 for k in ("back", "red"))
        return h2d, d2h


def gpu_uuid(device) -> str | None:
    try:
        u = str(torch.cuda.get_device_properties(device).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return None


def barrier(local):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier(device_ids=[local])
    torch.cuda.synchronize()


def run_gpu(args):
    import torch.distributed as dist
    rank, world, local = dist_env()
    if args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=device)
    step = Step(device)
    stream = torch.cuda.current_stream(device)

    # warm-up (untimed) and a correctness check of the buffers the bench times
    for _ in range(args.warmup):
        step.run(stream=stream)
    torch.cuda.synchronize()
    if not step.verify():
        raise SystemExit("bench step produced wrong results")

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    launches = 0
    with ClockSampler(gpu_uuid(device)) as clocks:
        barrier(local)
        start.record(stream)
        for k in range(K):
            launches += step.run(events=evs[k], stream=stream)
        end.record(stream)
        barrier(local)
    elapsed = start.elapsed_time(end) / 1e3
    per_kernel_s = {"seq_to_head": 0.0, "head_to_seq": 0.0, "ragged_reduce_scatter": 0.0}
    for e in evs:
        per_kernel_s["seq_to_head"] += e[0].elapsed_time(e[1]) / 1e3
        per_kernel_s["head_to_seq"] += e[1].elapsed_time(e[2]) / 1e3
        per_kernel_s["ragged_reduce_scatter"] += e[2].elapsed_time(e[3]) / 1e3
    t_max = max_over_ranks(elapsed, device)
    launches_total = int(sum_over_ranks(launches, device))
    value = throughput_gbs(step.bytes_per_step, K, world, t_max)
    peak, peak_kind = load_peak()

    kernels = {}
    for name, secs in per_kernel_s.items():
        n_launch = step.launches[name] * K
        per_launch_s = secs / n_launch
        bytes_per_launch = step.kernel_bytes[name] / step.launches[name]
        kernels[name] = {"gbs": round(bytes_per_launch / per_launch_s / 1e9, 1),
                         "us_per_launch": round(per_launch_s * 1e6, 2),
                         "launches_per_step": step.launches[name],
                         "bytes_per_launch": int(bytes_per_launch),
                         "share": round(secs / sum(per_kernel_s.values()), 3)}
    dom = max(kernels, key=lambda k: kernels[k]["share"])
    achieved = kernels[dom]["gbs"]
    roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak,
                "unit": "GB/s", "frac": round(achieved / peak, 4),
                "peak_source": f"{peak_kind}: MEASURED_PEAKS.json hbm_gbs" if peak_kind == "measured"
                else "fallback 6650 GB/s",
                "traffic": load_traffic(dom), "algorithmic_bytes_per_launch": kernels[dom]["bytes_per_launch"]}

    # end to end through the public API with pinned host buffers: every step
    # copies its inputs in and its results out.  Two device buffer sets and
    # three streams (host->device, compute, device->host) ordered by events
    # let step k's result copy and step k+1's input copy overlap the kernels.
    e2e = None
    if args.e2e_steps > 0:
        io = step.host_io()
        h2d, d2h = Step.io_bytes(io)
        bufs = [step, Step(device)]
        s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        loaded = [torch.cuda.Event() for _ in bufs]
        computed = [torch.cuda.Event() for _ in bufs]
        unloaded = [torch.cuda.Event() for _ in bufs]

        def e2e_step(k):
            b = k % 2
            st = bufs[b]
            if k >= 2:
                s_in.wait_event(computed[b])      # step k-2 is done reading this buffer set
            with torch.cuda.stream(s_in):
                st.qkv.copy_(io["qkv"], non_blocking=True)
                st.partials.copy_(io["partials"], non_blocking=True)
                st.bias.copy_(io["bias"], non_blocking=True)
                loaded[b].record(s_in)
            s_run.wait_event(loaded[b])
            if k >= 2:
                s_run.wait_event(unloaded[b])     # step k-2's results have left this buffer set
            n = st.run(stream=s_run)
            computed[b].record(s_run)
            s_out.wait_event(computed[b])
            with torch.cuda.stream(s_out):
                io["back"].copy_(st.back_full, non_blocking=True)
                io["red"].copy_(st.red_full, non_blocking=True)
                unloaded[b].record(s_out)
            return n

        for k in range(2):                        # warm both buffer sets
            e2e_step(k)
        torch.cuda.synchronize()
        barrier(local)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        s_run.wait_stream(s_in)
        s_out.wait_stream(s_in)
        for k in range(args.e2e_steps):
            e2e_step(k + 2)
        s_in.wait_stream(s_run)
        s_in.wait_stream(s_out)
        e1.record(s_in)
        barrier(local)
        t_e2e = max_over_ranks(e0.elapsed_time(e1) / 1e3, device)
        ok = torch.equal(io["back"].view(torch.int16), io["qkv"].view(torch.int16))
        e2e = {"value": round(throughput_gbs(step.bytes_per_step, args.e2e_steps, world, t_e2e), 2),
               "unit": UNIT, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": args.e2e_steps, "ms_per_step": round(t_e2e / args.e2e_steps * 1e3, 3),
               "mode": "pinned host buffers; copies in, kernels and copies out on three streams, "
                       "two device buffer sets",
               "round_trip_ok": bool(ok)}
        del io, bufs

    result = None
    if rank == 0:
        result = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": round(t_max / K * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "h3_transport_step_T32768_W6", "tokens": STEP_T,
                       "planes": STEP_P, "heads": wl.H3_HEADS, "head_dim": wl.H3_HEAD_DIM,
                       "world": STEP_W, "segments": STEP_SEGS, "reduce_cols": wl.H3_HIDDEN,
                       "window_bytes": WINDOW, "parallelism": f"replicas x{world}",
                       "l2": "no flush: every kernel's inputs (1.4-2.8 GB) exceed the 126 MB L2",
                       "bytes_per_step": step.bytes_per_step},
            "pct_of_peak": round(100.0 * value / world / peak, 2),
            "pct_of_nominal_peak": {"value": round(100.0 * value / world / NOMINAL_HBM_GBS, 2),
                                    "peak_gbs": NOMINAL_HBM_GBS,
                                    "source": "nominal B200 HBM3e bandwidth, ~8 TB/s"},
            "roofline": roofline,
            "kernels": kernels,
            "gpu_launches": launches_total,
            "clocks": clocks.summary(),
            "e2e": e2e,
            "library": os.path.relpath(step.rr.library_path, ROOT),
        }
    del step
    torch.cuda.empty_cache()
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    return result


# ---------------------------------------------------------------------------
# the oracle on the host cores
# ---------------------------------------------------------------------------

class OracleStep:
    """The same step through the CPU oracle on a token sample of the workload."""

    def __init__(self, tokens: int, W=STEP_W, P=STEP_P, seed=STEP_SEED):
        import oracle
        self.o = oracle.load()
        self.T, self.W, self.P, self.H, self.D, self.C = tokens, W, P, wl.H3_HEADS, wl.H3_HEAD_DIM, wl.H3_HIDDEN
        self.bounds = wl.segment_bounds(tokens, min(STEP_SEGS, tokens), seed)
        full = wl.bf16_bits(wl.normal_bf16((tokens, P, self.H, self.D), seed))
        ts = self.o.partition_range(tokens, W)
        self.send = [full[ts[r]:ts[r + 1]] for r in range(W)]
        rw = wl.ReduceWorkload("sample", T=tokens, C=self.C, W=W, seed=seed + 100)
        partials, bias = wl.partials_and_bias(rw, "cpu")
        self.partials = [wl.bf16_bits(p) for p in partials.unbind(0)]
        self.bias = wl.bf16_bits(bias)
        self.bytes = tokens * P * self.H * self.D * 2 * 2 * 2 + (W + 1) * tokens * self.C * 2 + self.C * 2

    def run(self):
        o = self.o
        ts = o.partition_range(self.T, self.W)
        for r in range(self.W):
            o.clip_segments(self.bounds, int(ts[r]), int(ts[r + 1]))
        heads = o.seq_to_head(self.send, self.T, self.P, self.H, self.D, self.W)
        o.head_to_seq(heads, self.T, self.P, self.H, self.D, self.W)
        o.ragged_reduce_scatter(self.partials, self.bias, self.W)


def oracle_seconds_per_token() -> float:
    s = OracleStep(256)
    t0 = time.perf_counter()
    s.run()
    return (time.perf_counter() - t0) / 256


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def host_cpu_model() -> str:
    """The host CPU's model name (Linux /proc/cpuinfo), or "unknown"."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


class OracleSteps:
    """The step through the unchanged oracle on every host core at once: one
    token sample per thread, run concurrently (the C oracle is called without
    the GIL, so the threads use separate cores)."""

    def __init__(self, tokens_each: int, threads: int):
        from concurrent.futures import ThreadPoolExecutor
        self.steps = [OracleStep(tokens_each) for _ in range(threads)]
        self.tokens_each = tokens_each
        self.bytes = sum(s.bytes for s in self.steps)
        self.pool = ThreadPoolExecutor(max_workers=threads)

    def run(self):
        list(self.pool.map(lambda s: s.run(), self.steps))

    def close(self):
        self.pool.shutdown()


# tokens of one thread's sample: bounds host memory (about 70 KB per token)
MAX_TOKENS_PER_THREAD = 2048


def cpu_baseline(budget_s: float = 12.0) -> dict:
    """The oracle on every host core (the reported value) and on one core
    (`one_core`), each on a bounded token sample of the bench step."""
    per_tok = oracle_seconds_per_token()
    # one core: the step on one sample, best of 2
    tokens = int(min(STEP_T, max(STEP_W, budget_s / 4 / per_tok)))
    s = OracleStep(tokens)
    times = []
    for _ in range(2):
        t0 = time.perf_counter()
        s.run()
        times.append(time.perf_counter() - t0)
    t1 = min(times)
    one = {"value": round(s.bytes / t1 / 1e9, 3), "unit": UNIT, "cores": 1, "kind": "oracle",
           "sample": f"the step on {tokens} of {STEP_T} tokens (W={STEP_W}, same shapes otherwise), "
                     f"best of 2, {t1:.2f} s each, single-threaded C oracle"}
    del s
    # every core: one sample per thread, repeated for about budget/2 seconds
    cores = host_cores()
    each = int(max(STEP_W, min(MAX_TOKENS_PER_THREAD, budget_s / 8 / per_tok)))
    steps = OracleSteps(each, cores)
    steps.run()  # warm
    n, t0 = 0, time.perf_counter()
    while n == 0 or time.perf_counter() - t0 < budget_s / 2:
        steps.run()
        n += 1
    t = time.perf_counter() - t0
    steps.close()
    return {"value": round(steps.bytes * n / t / 1e9, 3), "unit": UNIT, "cores": cores,
            "kind": "oracle",
            "sample": f"{cores} threads, each the step on its own {each} tokens (W={STEP_W}, "
                      f"same shapes otherwise), {n} rounds in {t:.1f} s, C oracle unchanged",
            "cpu_model": host_cpu_model(), "one_core": one}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    budget = float(args.reference_budget)  # seconds for warm-up + timed steps
    per_tok = oracle_seconds_per_token()
    per_step = budget / max(1, args.steps + args.warmup)
    cores = host_cores()
    each = int(min(MAX_TOKENS_PER_THREAD, max(STEP_W, per_step / per_tok)))
    s = OracleSteps(each, cores)
    for _ in range(args.warmup):
        s.run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        s.run()
    t = time.perf_counter() - t0
    s.close()
    value = s.bytes * args.steps / t / 1e9
    sample = (f"each step: {cores} threads, each the path on its own {each} tokens (W={STEP_W}, "
              f"same shapes otherwise), C oracle unchanged")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(t / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "h3_transport_step_T32768_W6", "tokens": STEP_T, "world": STEP_W,
                   "sample_tokens": each * cores},
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample, "cpu_model": host_cpu_model()},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def run_profile(args):
    """Run one kernel of the path --steps times (for ncu captures); no timing.
    The step's kernels on the bench workload, and the widened rows on the same
    shapes: gated reduce-scatter (8 segments), all-gather of the reduce
    outputs, staged seq->head through the 896,000,000-byte window, and rank
    0's pulled seq->head share."""
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    T = args.profile_tokens
    relayout = args.profile in ("seq_to_head", "head_to_seq", "staged_seq_to_head", "rank_seq_to_head")
    step = Step(device, T=T, relayout=relayout, reduce=not relayout)
    rr = step.rr
    if args.profile == "head_to_seq":
        rr.seq_to_head(step.send, step.heads)
    extra = {}
    if args.profile == "gated_reduce_scatter":
        extra["gate"] = wl.normal_bf16((STEP_SEGS, step.C), STEP_SEED + 2, 1.0, device)
        extra["x_full"], extra["x"] = rr.alloc_reduce_outputs(T, step.C, step.W, device)
        extra["x_full"].copy_(wl.normal_bf16((T, step.C), STEP_SEED + 3, 1.0, device))
    elif args.profile == "all_gather":
        rr.ragged_reduce_scatter(step.partial_list, step.bias, step.red_out)
        extra["outs"] = [torch.empty((T, step.C), dtype=torch.bfloat16, device=device)
                         for _ in range(step.W)]
    elif args.profile == "staged_seq_to_head":
        extra["win"] = torch.empty(WINDOW, dtype=torch.uint8, device=device)
    elif args.profile == "rank_seq_to_head":
        extra["mine"] = torch.empty_like(step.heads[0])
    launches = 0
    for _ in range(args.steps):
        if args.profile == "seq_to_head":
            info = rr.seq_to_head(step.send, step.heads)
        elif args.profile == "head_to_seq":
            info = rr.head_to_seq(step.heads, step.back, window_bytes=WINDOW)
        elif args.profile == "reduce_scatter":
            info = rr.ragged_reduce_scatter(step.partial_list, step.bias, step.red_out)
        elif args.profile == "gated_reduce_scatter":
            info = rr.ragged_reduce_scatter_gated(step.partial_list, step.bias, extra["gate"],
                                                  step.bounds, extra["x"], step.red_out)
        elif args.profile == "all_gather":
            info = rr.ragged_all_gather(step.red_out, extra["outs"])
        elif args.profile == "staged_seq_to_head":
            info = rr.seq_to_head_staged(step.send, step.heads, extra["win"])
        else:
            info = rr.seq_to_head_rank(step.send, extra["mine"], 0, n_heads=step.H)
        launches += info["launches"]
    torch.cuda.synchronize()
    print(json.dumps({"profile": args.profile, "tokens": T, "launches": launches}), flush=True)
    return 0


def _time_calls(fn, iters: int, warmup: int = 3) -> float:
    """Average device seconds per call of fn() (back-to-back on one stream)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        fn()
    e1.record()
    e1.synchronize()
    return e0.elapsed_time(e1) / 1e3 / iters


def run_workload_report(args):
    """Every kernel of the path on every workload, each variant: one JSON line
    per (workload, call, variant) with GB/s and the fraction of the peak."""
    import ragged_reduce_b200 as rr
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    peak, peak_kind = load_peak()
    iters = max(3, args.steps)
    lines = []

    def emit(workload, call, variant, nbytes, secs, info):
        rec = {"workload": workload, "call": call, "variant": variant,
               "gbs": round(nbytes / secs / 1e9, 1), "us": round(secs * 1e6, 1),
               "frac_of_" + peak_kind: round(nbytes / secs / 1e9 / peak, 4),
               "bytes": nbytes, "launches": info["launches"], "grid": info["grid"],
               "block": info["block"]}
        lines.append(rec)
        print(json.dumps(rec), flush=True)

    variants = [("default", 0), ("vector", rr.H3_VARIANT_VECTOR), ("bulk", rr.H3_VARIANT_BULK)]
    for w in (wl.TINY_QKV_W2, wl.QKV_32K_W6, wl.QKVG_128K_W4, wl.QKVG_250K_W4_CHUNKED):
        x = wl.packed_operand(w, device=dev)
        part = rr.partition(w.T, w.H, w.W)
        send = rr.split_rows(x, part.token_starts)
        heads = rr.alloc_head_side(w.T, w.P, w.H, w.D, w.W, dev)
        back_full, back = rr.alloc_seq_side(w.T, w.P, w.H, w.D, w.W, dev)
        nbytes = 2 * x.numel() * 2
        for vname, v in variants:
            info = rr.seq_to_head(send, heads, window_bytes=w.window_bytes, variant=v)
            secs = _time_calls(lambda: rr.seq_to_head(send, heads, window_bytes=w.window_bytes,
                                                      variant=v), iters)
            emit(w.name, "seq_to_head", vname, nbytes, secs, info)
            info = rr.head_to_seq(heads, back, window_bytes=w.window_bytes, variant=v)
            secs = _time_calls(lambda: rr.head_to_seq(heads, back, window_bytes=w.window_bytes,
                                                      variant=v), iters)
            emit(w.name, "head_to_seq", vname, nbytes, secs, info)
            if not torch.equal(back_full.view(torch.int16), x.view(torch.int16)):
                raise SystemExit(f"{w.name} {vname}: round trip differs")
        if w.T in (32768, 131072):
            # one rank per GPU, all W ranks' shares on this GPU back to back
            # (the same bytes as the one-GPU call)
            def s2h_ranks():
                for k in range(w.W):
                    last = rr.seq_to_head_rank(send, heads[k], k, n_heads=w.H,
                                               window_bytes=w.window_bytes)
                return last

            def h2s_ranks():
                for k in range(w.W):
                    last = rr.head_to_seq_rank(heads, back[k], k, n_tokens=w.T,
                                               window_bytes=w.window_bytes)
                return last

            for call, fn in (("seq_to_head", s2h_ranks), ("head_to_seq", h2s_ranks)):
                info = dict(fn())
                info["launches"] *= w.W
                secs = _time_calls(fn, iters)
                emit(w.name, call, "rank_shares", nbytes, secs, info)
            if not torch.equal(back_full.view(torch.int16), x.view(torch.int16)):
                raise SystemExit(f"{w.name} rank shares: round trip differs")
        if w.T < 32768:
            # small case: host overhead per call dominates; a prepared call
            # (checks and marshalling done once) and CUDA-graph replay
            fwd = rr.prepare_seq_to_head(send, heads, window_bytes=w.window_bytes)
            fwd()  # warm
            secs = _time_calls(fwd, iters * 10)
            emit(w.name, "seq_to_head", "prepared", nbytes, secs, rr.seq_to_head(send, heads))
            graph = torch.cuda.CUDAGraph()
            side = torch.cuda.Stream()
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                fwd()
            torch.cuda.current_stream().wait_stream(side)
            with torch.cuda.graph(graph):
                for _ in range(20):
                    fwd()
            secs = _time_calls(graph.replay, iters) / 20
            emit(w.name, "seq_to_head", "graph_replay", nbytes, secs, rr.seq_to_head(send, heads))
            del graph
        if w.T >= 32768:
            # staged through the pages' 896,000,000-byte window: every byte
            # crosses HBM twice, GB/s still counts the algorithmic bytes once
            win = torch.empty(min(WINDOW, 2 * x.numel()), dtype=torch.uint8, device=dev)
            info = rr.seq_to_head_staged(send, heads, win)
            secs = _time_calls(lambda: rr.seq_to_head_staged(send, heads, win), max(3, iters // 4))
            emit(w.name, "seq_to_head", "staged_896MB", nbytes, secs, info)
            info = rr.head_to_seq_staged(heads, back, win)
            secs = _time_calls(lambda: rr.head_to_seq_staged(heads, back, win), max(3, iters // 4))
            emit(w.name, "head_to_seq", "staged_896MB", nbytes, secs, info)
            if not torch.equal(back_full.view(torch.int16), x.view(torch.int16)):
                raise SystemExit(f"{w.name} staged: round trip differs")
            del win
        if w.inverse_planes:
            # head->seq on the attention output [T, 1, H, D]
            del heads, back_full, back
            torch.cuda.empty_cache()
            heads1 = [wl.normal_bf16((w.T, 1, part.heads(j), w.D), w.seed + 10 + j, 1.0, dev)
                      for j in range(w.W)]
            out_full, out = rr.alloc_seq_side(w.T, 1, w.H, w.D, w.W, dev)
            nb1 = 2 * out_full.numel() * 2
            for vname, v in variants:
                info = rr.head_to_seq(heads1, out, variant=v)
                secs = _time_calls(lambda: rr.head_to_seq(heads1, out, variant=v), iters)
                emit(w.name + "_attn_out", "head_to_seq", vname, nb1, secs, info)
            del heads1, out_full, out
        else:
            del heads, back_full, back
        del x, send
        torch.cuda.empty_cache()
    for rw in (wl.RS_64K_W8, wl.ReduceWorkload("reduce_scatter_T32768_C7168_W6", T=32768,
                                               C=wl.H3_HIDDEN, W=6, seed=102)):
        partials, bias = wl.partials_and_bias(rw, dev)
        plist = list(partials.unbind(0))
        out_full, out = rr.alloc_reduce_outputs(rw.T, rw.C, rw.W, dev)
        nbytes = (rw.W + 1) * rw.T * rw.C * 2 + rw.C * 2
        info = rr.ragged_reduce_scatter(plist, bias, out)
        secs = _time_calls(lambda: rr.ragged_reduce_scatter(plist, bias, out), iters)
        emit(rw.name, "ragged_reduce_scatter", "default", nbytes, secs, info)
        want = out_full.clone()

        def rs_ranks():
            for k in range(rw.W):
                last = rr.ragged_reduce_scatter_rank(plist, bias, out[k], k, n_tokens=rw.T)
            return last

        info = dict(rs_ranks())
        info["launches"] *= rw.W
        secs = _time_calls(rs_ranks, iters)
        emit(rw.name, "ragged_reduce_scatter", "rank_shares", nbytes, secs, info)
        if not torch.equal(out_full.view(torch.int16), want.view(torch.int16)):
            raise SystemExit(f"{rw.name}: rank shares differ from the one-GPU call")
        del partials, bias, plist, out_full, out, want
        torch.cuda.empty_cache()
    for rw, S in ((wl.RS_64K_W8, 16), (wl.ReduceWorkload("reduce_scatter_T32768_C7168_W6", T=32768,
                                                          C=wl.H3_HIDDEN, W=6, seed=102), 8)):
        partials, bias = wl.partials_and_bias(rw, dev)
        plist = list(partials.unbind(0))
        gate = wl.normal_bf16((S, rw.C), rw.seed + 2, 1.0, dev)
        bounds = wl.segment_bounds(rw.T, S, rw.seed)
        x_full, x = rr.alloc_reduce_outputs(rw.T, rw.C, rw.W, dev)
        x_full.copy_(wl.normal_bf16((rw.T, rw.C), rw.seed + 3, 1.0, dev))
        out_full, out = rr.alloc_reduce_outputs(rw.T, rw.C, rw.W, dev)
        nbytes = (rw.W + 2) * rw.T * rw.C * 2 + (S + 1) * rw.C * 2
        info = rr.ragged_reduce_scatter_gated(plist, bias, gate, bounds, x, out)
        secs = _time_calls(lambda: rr.ragged_reduce_scatter_gated(plist, bias, gate, bounds, x, out),
                           iters)
        emit(rw.name.replace("reduce_scatter", "gated_reduce_scatter"), "ragged_reduce_scatter_gated",
             "default", nbytes, secs, info)
        del partials, bias, plist, gate, x_full, x, out_full, out
        torch.cuda.empty_cache()
    for (T, C_, W) in ((65536, wl.H3_HIDDEN, 8), (32768, wl.H3_HIDDEN, 6)):
        full = wl.normal_bf16((T, C_), 9, 1.0, dev)
        blocks = rr.split_rows(full, rr.partition(T, W, W).token_starts)
        outs = [torch.empty((T, C_), dtype=torch.bfloat16, device=dev) for _ in range(W)]
        nbytes = (1 + W) * T * C_ * 2
        info = rr.ragged_all_gather(blocks, outs)
        secs = _time_calls(lambda: rr.ragged_all_gather(blocks, outs), iters)
        emit(f"all_gather_T{T}_C{C_}_W{W}", "ragged_all_gather", "default", nbytes, secs, info)
        if not all(torch.equal(o.view(torch.int16), full.view(torch.int16)) for o in outs):
            raise SystemExit("all-gather output differs")
        for o in outs:
            o.zero_()

        def ag_ranks():
            for k in range(W):
                last = rr.ragged_all_gather_rank(blocks, outs[k], k)
            return last

        info = dict(ag_ranks())
        info["launches"] *= W
        secs = _time_calls(ag_ranks, iters)
        emit(f"all_gather_T{T}_C{C_}_W{W}", "ragged_all_gather", "rank_shares", nbytes, secs, info)
        if not all(torch.equal(o.view(torch.int16), full.view(torch.int16)) for o in outs):
            raise SystemExit("all-gather rank shares differ")
        del full, blocks, outs
        torch.cuda.empty_cache()
    if rr.bulk_wait_timeouts() != 0:
        raise SystemExit("bulk kernel reported expired waits")
    return 0


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=1000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["native", "reference"], default="native")
    p.add_argument("--e2e-steps", type=int, default=16)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-budget", type=float, default=12.0,
                   help="about how many seconds cpu_baseline spends on the oracle")
    p.add_argument("--profile", choices=["seq_to_head", "head_to_seq", "reduce_scatter",
                                         "gated_reduce_scatter", "all_gather",
                                         "staged_seq_to_head", "rank_seq_to_head"],
                   help="run only this kernel of the step --steps times (ncu captures); no timing")
    p.add_argument("--profile-tokens", type=int, default=STEP_T)
    p.add_argument("--report-workloads", action="store_true",
                   help="time every kernel and variant on every workload (one JSON line each)")
    p.add_argument("--reference-budget", type=float, default=90.0,
                   help="seconds of oracle work for --impl reference (warm-up + timed)")
    return p.parse_args(argv)


def main(argv=None):
    args = parse_args(argv)
    if args.profile:
        return run_profile(args)
    if args.report_workloads:
        return run_workload_report(args)
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.impl == "reference":
        result = run_reference(args)
        if result is not None:
            print(json.dumps(result), flush=True)
        return 0
    result = run_gpu(args)
    if result is not None:
        rank, world, _ = dist_env()
        if world == 1 and not args.no_cpu_baseline:
            result["cpu_baseline"] = cpu_baseline(budget_s=args.cpu_budget)
        else:
            result["cpu_baseline"] = None
        print(json.dumps(result), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
