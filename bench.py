#!/usr/bin/env python
"""Benchmark of the H3 transport hot path on B200: effective HBM GB/s.

One step is one pass of the whole path over the two largest workloads of the
path:

  1. h3_partition             token/head ranges, packed segments clipped and rebased (host)
  2. h3_seq_to_head           packed QKVG [250000, 4, 56, 128] over W = 4 ranks (heads
                              14 each) -> 4 x [250000, 4, 14, 128], one batch plane
                              per launch under the 896,000,000-byte window (4 launches)
  3. h3_head_to_seq           back to [250000, 4, 56, 128], chunked the same way
  4. h3_ragged_reduce_scatter 8 BF16 partials [65536, 7168] + bias -> 8 x [8192, 7168]

value = algorithmic bytes of all steps (each input read once + each output
written once) / device time.  Every kernel's inputs are 7.2-15 GB, far larger
than the 126 MB L2, so no flush is needed between steps.

With --gpus N > 1 (torchrun, one process per GPU) the same two problems run
with one rank per GPU (W = N): every GPU holds its rank's buffers only and
computes its rank's share with the h3_*_rank calls, pulling what it needs
from the peers' buffers (mapped with CUDA IPC) over NVLink; a one-element
NCCL all-reduce on the compute stream orders the ranks between the calls.
The total problem is fixed as N grows (strong scaling).

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
# The step's two problems: the long-sequence QKVG round trip, one batch plane
# per launch under the 896,000,000-byte window, and the 8-way reduce-scatter.
RELAYOUT = wl.QKVG_250K_W4_CHUNKED
REDUCE = wl.RS_64K_W8
WINDOW = RELAYOUT.window_bytes
WORKLOAD = f"{RELAYOUT.name}+{REDUCE.name}"


# ---------------------------------------------------------------------------
# host-side helpers (no GPU needed; covered by the gloo tests)
# ---------------------------------------------------------------------------

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def _reduce_over_ranks(x: float, device, op) -> float:
    """x reduced over all ranks with `op` (x itself without a process group);
    gloo reduces a host tensor, NCCL one on `device`."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    dev = device if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(x: float, device) -> float:
    """Largest value of x over all ranks (x itself without a process group)."""
    import torch.distributed as dist
    return _reduce_over_ranks(x, device, dist.ReduceOp.MAX)


def sum_over_ranks(x: float, device) -> float:
    import torch.distributed as dist
    return _reduce_over_ranks(x, device, dist.ReduceOp.SUM)


def min_over_ranks(x: float, device) -> float:
    """Smallest value of x over all ranks (x itself without a process group)."""
    import torch.distributed as dist
    return _reduce_over_ranks(x, device, dist.ReduceOp.MIN)


def throughput_gbs(bytes_per_step_per_gpu: float, steps: int, n_gpus: int, seconds: float) -> float:
    """Whole-job GB/s: every GPU's bytes over the slowest GPU's time."""
    return bytes_per_step_per_gpu * steps * n_gpus / seconds / 1e9


def step_bytes(world: int) -> int:
    """Whole-job algorithmic bytes of one step: the QKVG round trip (every
    element read and written once each way) and the reduce-scatter; with one
    rank per GPU every rank also reads the bias."""
    rb = relayout_bytes(RELAYOUT.T, RELAYOUT.P, RELAYOUT.H, RELAYOUT.D)
    if world > 1:
        return 2 * rb + reduce_bytes(REDUCE.T, REDUCE.C, world) + (world - 1) * REDUCE.C * 2
    return 2 * rb + reduce_bytes(REDUCE.T, REDUCE.C, REDUCE.W)


def step_config(world: int) -> dict:
    """The line's `config`: the workload the step runs at `world` GPUs, the
    same for the native and the reference arm."""
    if world > 1:
        parallelism = (f"one rank per GPU: W={world} ranks, tokens and heads split "
                       f"by quotient/remainder, shares pulled over NVLink")
    else:
        parallelism = (f"one GPU: W={RELAYOUT.W} virtual ranks (relayout), "
                       f"W={REDUCE.W} (reduce-scatter)")
    return {"workload": WORKLOAD,
            "relayout": {"tokens": RELAYOUT.T, "planes": RELAYOUT.P,
                         "heads": RELAYOUT.H, "head_dim": RELAYOUT.D,
                         "world": world if world > 1 else RELAYOUT.W,
                         "segments": RELAYOUT.n_segs, "window_bytes": WINDOW,
                         "chunking": "one batch plane per launch"},
            "reduce_scatter": {"tokens": REDUCE.T, "cols": REDUCE.C,
                               "world": world if world > 1 else REDUCE.W,
                               "partial_std": REDUCE.partial_std,
                               "bias_std": REDUCE.bias_std},
            "parallelism": parallelism,
            "l2": "no flush: every kernel's inputs (7.2-15 GB) exceed the 126 MB L2",
            "bytes_per_step": step_bytes(world)}


def load_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# The sources each measured kernel is compiled from (the rank calls' pull
# kernel lives in relayout.cu too).
KERNEL_SOURCES = {
    "seq_to_head": ("relayout.cu", "device_access.cuh", "bulk_copy.cuh", "kernel_args.h"),
    "head_to_seq": ("relayout.cu", "device_access.cuh", "bulk_copy.cuh", "kernel_args.h"),
    "ragged_reduce_scatter": ("reduce_scatter.cu", "bf16_sum.cuh", "device_access.cuh", "kernel_args.h"),
}


def kernel_source_digest(kernel: str) -> str:
    """Digest of the sources `kernel` is compiled from: traffic figures taken
    with other sources are not reported."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "ragged_reduce_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_traffic(kernel: str, instance: str | None = None):
    """DRAM bytes per launch of `kernel` on the launches `instance` names,
    from the committed ncu summary; None when no capture covers that
    instance or the kernel's sources changed since it was taken."""
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
            table = json.load(f)
    except (OSError, ValueError):
        return None
    entry = table.get(kernel)
    if not entry or kernel not in KERNEL_SOURCES or entry.get("source_digest") != kernel_source_digest(kernel):
        return None
    if instance is not None and entry.get("instance") != instance:
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

KERNELS = ("seq_to_head", "head_to_seq", "ragged_reduce_scatter")


def relayout_bytes(T: int, P: int, H: int, D: int) -> int:
    """Algorithmic bytes of one relayout direction: every element read once
    and written once."""
    return 2 * T * P * H * D * 2


def reduce_bytes(T: int, C: int, W: int) -> int:
    """Algorithmic bytes of the reduce-scatter: W partials read, the [T, C]
    output written, the bias read once."""
    return (W + 1) * T * C * 2 + C * 2


class Step:
    """Device buffers and calls of one step of the path on one GPU, with all
    W virtual ranks in its memory (inputs resident).  tokens / rows shrink the
    two problems (ncu captures of small cases); relayout / reduce leave one out."""

    def __init__(self, device, *, tokens=None, rows=None, relayout=True, reduce=True):
        import ragged_reduce_b200 as rr
        self.rr = rr
        self.device = device
        rw, red = RELAYOUT, REDUCE
        self.T, self.P, self.W, self.H, self.D = tokens or rw.T, rw.P, rw.W, rw.H, rw.D
        self.window = rw.window_bytes
        self.Tr, self.C, self.Wr = rows or red.T, red.C, red.W
        self.bounds = wl.segment_bounds(self.T, rw.n_segs, rw.seed)
        self.kernel_bytes = {}
        self.has_relayout, self.has_reduce = relayout, reduce
        if relayout:
            self.part = rr.partition(self.T, self.H, self.W, self.bounds)
            self.qkv = wl.normal_bf16((self.T, self.P, self.H, self.D), rw.seed, 1.0, device)
            self.send = rr.split_rows(self.qkv, self.part.token_starts)
            self.heads = rr.alloc_head_side(self.T, self.P, self.H, self.D, self.W, device)
            self.back_full, self.back = rr.alloc_seq_side(self.T, self.P, self.H, self.D, self.W, device)
            b = relayout_bytes(self.T, self.P, self.H, self.D)
            self.kernel_bytes["seq_to_head"] = b
            self.kernel_bytes["head_to_seq"] = b
        if reduce:
            w = wl.ReduceWorkload(red.name, T=self.Tr, C=self.C, W=self.Wr, seed=red.seed)
            self.partials, self.bias = wl.partials_and_bias(w, device)
            self.partial_list = list(self.partials.unbind(0))
            self.red_full, self.red_out = rr.alloc_reduce_outputs(self.Tr, self.C, self.Wr, device)
            self.kernel_bytes["ragged_reduce_scatter"] = reduce_bytes(self.Tr, self.C, self.Wr)
        self.bytes_per_step = sum(self.kernel_bytes.values())
        self.launches = {}

    def instance(self, kernel: str) -> str:
        """The launches `kernel` makes in this step, as ncu summaries name them."""
        if kernel == "ragged_reduce_scatter":
            return f"reduce_scatter T={self.Tr} C={self.C} W={self.Wr}"
        return (f"{kernel} T={self.T} P={self.P} W={self.W} one plane per launch "
                f"(window {self.window})")

    def run(self, events=None, stream=None):
        """Enqueue one step; events[0..3] (optional) bracket the three calls."""
        rr = self.rr

        def mark(i):
            if events is not None:
                events[i].record(stream)

        mark(0)
        infos = {}
        if self.has_relayout:
            rr.partition(self.T, self.H, self.W, self.bounds)
            infos["seq_to_head"] = rr.seq_to_head(self.send, self.heads, window_bytes=self.window,
                                                  stream=stream)
        mark(1)
        if self.has_relayout:
            infos["head_to_seq"] = rr.head_to_seq(self.heads, self.back, window_bytes=self.window,
                                                  stream=stream)
        mark(2)
        if self.has_reduce:
            infos["ragged_reduce_scatter"] = rr.ragged_reduce_scatter(self.partial_list, self.bias,
                                                                      self.red_out, stream=stream)
        mark(3)
        self.launches = {k: v["launches"] for k, v in infos.items()}
        return sum(self.launches.values())

    def verify(self) -> bool:
        """Round trip and reduce check on the device with torch (not timed)."""
        ok = True
        if self.has_relayout:
            ok = torch.equal(self.back_full.view(torch.int16), self.qkv.view(torch.int16))
        if self.has_reduce:
            acc = self.partials[0].float()
            for k in range(1, self.Wr):
                acc += self.partials[k].float()
            acc += self.bias.float()
            ok = ok and torch.equal(self.red_full.view(torch.int16),
                                    acc.to(torch.bfloat16).view(torch.int16))
            del acc
        return bool(ok)

    def inputs(self) -> dict:
        """Device tensors a caller fills from the host every step."""
        return {"qkv": self.qkv, "partials": self.partials, "bias": self.bias}

    def outputs(self) -> dict:
        """Device tensors a caller reads back every step."""
        return {"back": self.back_full, "red": self.red_full}

    def nvlink(self, per_kernel_s: dict, steps: int):
        return None

    def token_range_rates(self, iters: int, stream) -> dict:
        """The step's two relayouts under the same window cut into token
        ranges of every plane (H3_LAUNCH_CHUNK_TOKENS) instead of one batch
        plane per launch: GB/s per direction by CUDA events over `iters`
        calls after two warm-up calls, and the round trip checked.  Not part
        of the bench's value."""
        rr = self.rr
        out = {}
        kw = dict(window_bytes=self.window, stream=stream, token_chunks=True)
        for name, call in (("seq_to_head", lambda: rr.seq_to_head(self.send, self.heads, **kw)),
                           ("head_to_seq", lambda: rr.head_to_seq(self.heads, self.back, **kw))):
            for _ in range(2):
                info = call()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(iters):
                call()
            e1.record(stream)
            e1.synchronize()
            secs = e0.elapsed_time(e1) / 1e3 / iters
            out[name] = {"gbs": round(self.kernel_bytes[name] / secs / 1e9, 1),
                         "us_per_call": round(secs * 1e6, 1), "launches_per_call": info["launches"],
                         "planes_per_launch": info["planes_per_launch"]}
        tokens, _ = rr.relayout_chunk_plan(self.T, self.P, self.H, self.D, self.W, self.window,
                                           token_chunks=True)
        out["tokens_per_launch"] = tokens
        out["round_trip_ok"] = bool(torch.equal(self.back_full.view(torch.int16),
                                                self.qkv.view(torch.int16)))
        return out


class ShardedStep:
    """One rank's share of the step with one rank per GPU (W = world).

    Each process holds its rank's buffers only: the sequence-side rows
    [T_k, P, H, D], the head-side buffer [T, P, H_k, D], the rows it gets back,
    its partial [T, C], the bias and its reduce-scatter rows [T_k, C].  The
    rank calls pull what rank k needs from every rank's buffer through the
    peer tables.  Between the calls `fence(stream)` orders all ranks (a
    one-element all-reduce enqueued on the compute stream): head->seq reads
    the peers' head-side buffers that seq->head has just written, and the next
    step's seq->head must not overwrite a head-side buffer a peer still reads.

    Injectable for host-side tests: `rr` (the binding's partition and rank
    calls), `peer_table` (tensor -> object with .pointers and .close()),
    `fence`, and `empty(shape, dtype)`, which allocates the three buffers the
    peers read (sequence-side rows, head-side buffer, partial)."""

    def __init__(self, device, rank: int, world: int, *, rr, peer_table, fence,
                 tokens=None, rows=None, empty=None):
        if empty is None:
            def empty(shape, dtype):
                return torch.empty(shape, dtype=dtype, device=device)
        self.rr, self.fence = rr, fence
        self.device, self.rank, self.W = device, rank, world
        rw, red = RELAYOUT, REDUCE
        self.T, self.P, self.H, self.D = tokens or rw.T, rw.P, rw.H, rw.D
        self.window = rw.window_bytes
        self.Tr, self.C = rows or red.T, red.C
        self.bounds = wl.segment_bounds(self.T, rw.n_segs, rw.seed)
        part = rr.partition(self.T, self.H, world, self.bounds)
        self.ts = (int(part.token_starts[rank]), int(part.token_starts[rank + 1]))
        self.hk = part.heads(rank)
        # the whole operand is drawn from the same seed as the one-GPU step;
        # this rank keeps its token rows
        x = wl.normal_bf16((self.T, self.P, self.H, self.D), rw.seed, 1.0, device)
        self.send = empty((self.ts[1] - self.ts[0], self.P, self.H, self.D), torch.bfloat16)
        self.send.copy_(x[self.ts[0]:self.ts[1]])
        del x
        self.heads = empty((self.T, self.P, self.hk, self.D), torch.bfloat16)
        self.back = torch.empty_like(self.send)
        w = wl.ReduceWorkload(red.name, T=self.Tr, C=self.C, W=world, seed=red.seed)
        partials, self.bias = wl.partials_and_bias(w, device)
        rp = rr.partition(self.Tr, world, world)
        self.rows = (int(rp.token_starts[rank]), int(rp.token_starts[rank + 1]))
        self.partial = empty((self.Tr, self.C), torch.bfloat16)
        self.partial.copy_(partials[rank])
        # every rank's rows of this rank's output, kept for verify()
        self.check_rows = partials[:, self.rows[0]:self.rows[1]].clone()
        del partials
        self.red_out = torch.empty((self.rows[1] - self.rows[0], self.C), dtype=torch.bfloat16,
                                   device=device)
        # collective: every rank builds the tables in the same order
        self.seq_tab = peer_table(self.send)
        self.head_tab = peer_table(self.heads)
        self.part_tab = peer_table(self.partial)
        # whole-job algorithmic bytes (every element read and written once;
        # each rank reads the bias once)
        rb = relayout_bytes(self.T, self.P, self.H, self.D)
        self.kernel_bytes = {"seq_to_head": rb, "head_to_seq": rb,
                             "ragged_reduce_scatter": reduce_bytes(self.Tr, self.C, world)
                             + (world - 1) * self.C * 2}
        self.bytes_per_step = sum(self.kernel_bytes.values())
        self.launches = {}

    def instance(self, kernel: str) -> str:
        return f"{kernel} rank share, one rank per GPU, W={self.W}"

    def run(self, events=None, stream=None):
        """Enqueue this rank's share of one step; events[0..4] (optional)
        bracket the calls, the fence after seq->head excluded."""
        rr, k = self.rr, self.rank

        def mark(i):
            if events is not None:
                events[i].record(stream)

        mark(0)
        rr.partition(self.T, self.H, self.W, self.bounds)
        i1 = rr.seq_to_head_rank(self.seq_tab.pointers, self.heads, k, n_heads=self.H,
                                 window_bytes=self.window, stream=stream)
        mark(1)
        self.fence(stream)  # every head-side buffer is complete before anyone reads it
        mark(2)
        i2 = rr.head_to_seq_rank(self.head_tab.pointers, self.back, k, n_tokens=self.T,
                                 window_bytes=self.window, stream=stream)
        mark(3)
        i3 = rr.ragged_reduce_scatter_rank(self.part_tab.pointers, self.bias, self.red_out, k,
                                           n_tokens=self.Tr, stream=stream)
        mark(4)
        self.fence(stream)  # no head-side buffer is overwritten while a peer reads it
        self.launches = {"seq_to_head": i1["launches"], "head_to_seq": i2["launches"],
                         "ragged_reduce_scatter": i3["launches"]}
        return sum(self.launches.values())

    def verify(self) -> bool:
        """This rank's round trip and its reduce rows, checked with torch."""
        ok = torch.equal(self.back.view(torch.int16), self.send.view(torch.int16))
        acc = self.check_rows[0].float()
        for r in range(1, self.W):
            acc += self.check_rows[r].float()
        acc += self.bias.float()
        return bool(ok and torch.equal(self.red_out.view(torch.int16),
                                       acc.to(torch.bfloat16).view(torch.int16)))

    def inputs(self) -> dict:
        return {"send": self.send, "partial": self.partial, "bias": self.bias}

    def outputs(self) -> dict:
        return {"back": self.back, "red": self.red_out}

    def pulled_bytes(self) -> dict:
        """Bytes this rank's calls read from other ranks' memory per step."""
        row = self.H * self.D * 2
        tk = self.ts[1] - self.ts[0]
        return {"seq_to_head": (self.T - tk) * self.P * self.hk * self.D * 2,
                "head_to_seq": tk * self.P * (row - self.hk * self.D * 2),
                "ragged_reduce_scatter": (self.W - 1) * (self.rows[1] - self.rows[0]) * self.C * 2}

    def nvlink(self, per_kernel_s: dict, steps: int):
        pulled = self.pulled_bytes()
        return {k: {"bytes_per_step": int(v),
                    "gbs": round(v * steps / per_kernel_s[k] / 1e9, 1) if per_kernel_s[k] > 0 else None}
                for k, v in pulled.items()}

    def close(self):
        for t in (self.seq_tab, self.head_tab, self.part_tab):
            t.close()


def gpu_uuid(device) -> str | None:
    try:
        u = str(torch.cuda.get_device_properties(device).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return None


class CudaTimer:
    """Device timestamps: CUDA events recorded on the launching stream."""

    def event(self):
        return torch.cuda.Event(enable_timing=True)

    @staticmethod
    def seconds(a, b) -> float:
        return a.elapsed_time(b) / 1e3

    @staticmethod
    def synchronize():
        torch.cuda.synchronize()


class _HostEvent:
    def __init__(self):
        self.t = None

    def record(self, stream=None):
        self.t = time.perf_counter()


class HostTimer:
    """Host timestamps for runs without a GPU (host-side tests)."""

    def event(self):
        return _HostEvent()

    @staticmethod
    def seconds(a, b) -> float:
        return b.t - a.t

    @staticmethod
    def synchronize():
        pass


def barrier(local, timer=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if dist.get_backend() == "nccl":
            dist.barrier(device_ids=[local])
        else:
            dist.barrier()
    (timer or CudaTimer()).synchronize()


def nccl_fence(device):
    """A stream-ordered barrier of all ranks: a one-element all-reduce
    enqueued on `stream` completes on a rank only after every rank's stream
    has reached it, so whatever each rank enqueued before it has finished."""
    import torch.distributed as dist
    token = torch.zeros(1, dtype=torch.int32, device=device)

    def fence(stream=None):
        if stream is None:
            dist.all_reduce(token)
        else:
            with torch.cuda.stream(stream):
                dist.all_reduce(token)
    return fence


def time_steps(step, K: int, timer, stream, local, n_events: int):
    """Run K steps between barriers; (seconds, launches, per-kernel seconds)."""
    evs = [[timer.event() for _ in range(n_events)] for _ in range(K)]
    start, end = timer.event(), timer.event()
    launches = 0
    barrier(local, timer)
    start.record(stream)
    for k in range(K):
        launches += step.run(events=evs[k], stream=stream)
    end.record(stream)
    barrier(local, timer)
    per_kernel_s = {name: 0.0 for name in KERNELS}
    # the events bracketing each call (the sharded step has a fence between
    # its first two calls, which no kernel's time includes)
    spans = ({"seq_to_head": (0, 1), "head_to_seq": (1, 2), "ragged_reduce_scatter": (2, 3)}
             if n_events == 4 else
             {"seq_to_head": (0, 1), "head_to_seq": (2, 3), "ragged_reduce_scatter": (3, 4)})
    for e in evs:
        for name, (a, b) in spans.items():
            per_kernel_s[name] += timer.seconds(e[a], e[b])
    return timer.seconds(start, end), launches, per_kernel_s


def kernel_table(step, per_kernel_s: dict, K: int) -> dict:
    kernels = {}
    total = sum(per_kernel_s.values())
    for name, secs in per_kernel_s.items():
        n = step.launches.get(name, 0)
        if n == 0 or secs <= 0:
            continue
        per_launch_s = secs / (n * K)
        bytes_per_launch = step.kernel_bytes[name] / n
        kernels[name] = {"gbs": round(bytes_per_launch / per_launch_s / 1e9, 1),
                         "us_per_launch": round(per_launch_s * 1e6, 2),
                         "launches_per_step": n,
                         "bytes_per_launch": int(bytes_per_launch),
                         "share": round(secs / total, 3),
                         "instance": step.instance(name)}
    return kernels


def run_e2e(make_step, first, n_steps: int, local, device, world: int, timer):
    """End to end through the public API with pinned host buffers: every step
    copies its inputs in and its results out.  Two device buffer sets and
    three streams (host->device, compute, device->host) ordered by events let
    step k's result copy and step k+1's input copy overlap the kernels."""
    ins = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in first.inputs().items()}
    for k, v in first.inputs().items():
        ins[k].copy_(v)
    outs = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in first.outputs().items()}
    h2d = sum(v.numel() * v.element_size() for v in ins.values())
    d2h = sum(v.numel() * v.element_size() for v in outs.values())
    bufs = [first, make_step()]
    s_in, s_run, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device), torch.cuda.Stream(device)
    loaded = [torch.cuda.Event() for _ in bufs]
    computed = [torch.cuda.Event() for _ in bufs]
    unloaded = [torch.cuda.Event() for _ in bufs]

    def e2e_step(k):
        b = k % 2
        st = bufs[b]
        if k >= 2:
            s_in.wait_event(computed[b])      # step k-2 is done reading this buffer set
        with torch.cuda.stream(s_in):
            for name, dst in st.inputs().items():
                dst.copy_(ins[name], non_blocking=True)
            loaded[b].record(s_in)
        s_run.wait_event(loaded[b])
        if k >= 2:
            s_run.wait_event(unloaded[b])     # step k-2's results have left this buffer set
        n = st.run(stream=s_run)
        computed[b].record(s_run)
        s_out.wait_event(computed[b])
        with torch.cuda.stream(s_out):
            for name, src in st.outputs().items():
                outs[name].copy_(src, non_blocking=True)
            unloaded[b].record(s_out)
        return n

    for k in range(2):                        # warm both buffer sets
        e2e_step(k)
    torch.cuda.synchronize()
    barrier(local, timer)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    s_run.wait_stream(s_in)
    s_out.wait_stream(s_in)
    for k in range(n_steps):
        e2e_step(k + 2)
    s_in.wait_stream(s_run)
    s_in.wait_stream(s_out)
    e1.record(s_in)
    barrier(local, timer)
    t_e2e = max_over_ranks(e0.elapsed_time(e1) / 1e3, device)
    # the link's own bound: the same copies, both directions at once, no kernels
    torch.cuda.synchronize()
    barrier(local, timer)
    c0 = torch.cuda.Event(enable_timing=True)
    c1 = torch.cuda.Event(enable_timing=True)
    c0.record(s_in)
    s_out.wait_stream(s_in)
    link_steps = 2
    for _ in range(link_steps):
        with torch.cuda.stream(s_in):
            for name, dst in bufs[0].inputs().items():
                dst.copy_(ins[name], non_blocking=True)
        with torch.cuda.stream(s_out):
            for name, src in bufs[1].outputs().items():
                outs[name].copy_(src, non_blocking=True)
    s_in.wait_stream(s_out)
    c1.record(s_in)
    barrier(local, timer)
    t_link = max_over_ranks(c0.elapsed_time(c1) / 1e3 / link_steps, device)
    # the round trip comes back unchanged (the last step's results, copied
    # again above from the same buffers)
    key_in, key_out = ("qkv", "back") if "qkv" in ins else ("send", "back")
    ok = torch.equal(outs[key_out].view(torch.int16), ins[key_in].view(torch.int16))
    ok = bool(min_over_ranks(1.0 if ok else 0.0, device) > 0)
    second = bufs[1]
    if hasattr(second, "close"):
        torch.cuda.synchronize()
        barrier(local, timer)
        second.close()
    del bufs
    return {"value": round(throughput_gbs(first.bytes_per_step, n_steps, 1, t_e2e), 2),
            "unit": UNIT,
            "h2d_bytes_per_step": int(sum_over_ranks(h2d, device)),
            "d2h_bytes_per_step": int(sum_over_ranks(d2h, device)),
            "steps": n_steps, "ms_per_step": round(t_e2e / n_steps * 1e3, 3),
            "link_bound_ms_per_step": round(t_link * 1e3, 3),
            "frac_of_link_bound": round(t_link / (t_e2e / n_steps), 3),
            "mode": "pinned host buffers; copies in, kernels and copies out on three streams, "
                    "two device buffer sets" + (f", {world} GPUs" if world > 1 else ""),
            "round_trip_ok": ok}


def run_gpu(args):
    import torch.distributed as dist
    rank, world, local = dist_env()
    if args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    timer = CudaTimer()
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=device)
    import ragged_reduce_b200 as rr
    if world > 1:
        from ragged_reduce_b200 import peers

        def make_step():
            return ShardedStep(device, rank, world, rr=rr, peer_table=peers.PeerBuffers,
                               fence=nccl_fence(device))
        n_events = 5
    else:
        def make_step():
            return Step(device)
        n_events = 4
    result = measure(args, make_step, rank, world, local, device, timer, n_events)
    torch.cuda.empty_cache()
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    return result


def measure(args, make_step, rank, world, local, device, timer, n_events):
    """Warm-up, correctness check, K timed steps, e2e; rank 0's JSON record."""
    step = make_step()
    stream = torch.cuda.current_stream(device) if isinstance(timer, CudaTimer) else None
    # warm-up (untimed) and a correctness check of the buffers the bench times
    for _ in range(args.warmup):
        step.run(stream=stream)
    timer.synchronize()
    ok = step.verify()
    if min_over_ranks(1.0 if ok else 0.0, device) <= 0:
        raise SystemExit("bench step produced wrong results")

    K = args.steps
    with ClockSampler(gpu_uuid(device) if isinstance(timer, CudaTimer) else None) as clocks:
        elapsed, launches, per_kernel_s = time_steps(step, K, timer, stream, local, n_events)
    t_max = max_over_ranks(elapsed, device)
    launches_total = int(sum_over_ranks(launches, device))
    value = throughput_gbs(step.bytes_per_step, K, 1, t_max)
    peak, peak_kind = load_peak()
    kernels = kernel_table(step, per_kernel_s, K)
    dom = max(kernels, key=lambda k: kernels[k]["share"])
    achieved = kernels[dom]["gbs"] / world  # per GPU: each GPU moves 1/W of the bytes
    roofline = {"bound": "hbm", "kernel": dom, "instance": kernels[dom]["instance"],
                "achieved": round(achieved, 1), "peak": peak,
                "unit": "GB/s", "frac": round(achieved / peak, 4),
                "peak_source": f"{peak_kind}: MEASURED_PEAKS.json hbm_gbs" if peak_kind == "measured"
                else "fallback 6650 GB/s",
                "traffic": load_traffic(dom, kernels[dom]["instance"]) if world == 1 else None,
                "algorithmic_bytes_per_launch": kernels[dom]["bytes_per_launch"] // world}
    nvlink = step.nvlink(per_kernel_s, K)

    e2e = None
    if args.e2e_steps > 0 and isinstance(timer, CudaTimer):
        e2e = run_e2e(make_step, step, args.e2e_steps, local, device, world, timer)

    # Beside the line, not in its value: the same window cut into token
    # ranges of every plane instead of one batch plane per launch.
    ranges = None
    if (world == 1 and isinstance(timer, CudaTimer) and getattr(step, "has_relayout", False)
            and not getattr(args, "no_chunk_shapes", False)):
        ranges = step.token_range_rates(max(3, min(20, K)), stream)
        if not ranges["round_trip_ok"]:
            raise SystemExit("token-range relayouts produced wrong results")

    result = None
    if rank == 0:
        config = step_config(world)
        config["bytes_per_step"] = step.bytes_per_step  # the workload's, unless a test shrank it
        result = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": round(t_max / K * 1e3, 4),
            "higher_is_better": True, "scaling": "strong" if world > 1 else "weak",
            "vs_baseline": None, "dtype": "bf16", "accumulate_dtype": "f32", "data": "synthetic",
            "config": config,
            "pct_of_peak": round(100.0 * value / world / peak, 2),
            "pct_of_nominal_peak": {"value": round(100.0 * value / world / NOMINAL_HBM_GBS, 2),
                                    "peak_gbs": NOMINAL_HBM_GBS,
                                    "source": "nominal B200 HBM3e bandwidth, ~8 TB/s"},
            "roofline": roofline,
            "kernels": kernels,
            "gpu_launches": launches_total,
            "clocks": clocks.summary(),
            "e2e": e2e,
            "library": os.path.relpath(step.rr.library_path, ROOT)
            if hasattr(step.rr, "library_path") else None,
        }
        if nvlink is not None:
            result["nvlink_rank0"] = nvlink
        if ranges is not None:
            result["chunk_shapes"] = {
                "window_bytes": WINDOW,
                "one_plane_per_launch": {k: {"gbs": kernels[k]["gbs"],
                                             "launches_per_call": kernels[k]["launches_per_step"]}
                                         for k in ("seq_to_head", "head_to_seq")},
                "token_ranges_all_planes": ranges,
                "note": "not part of value: the step's relayouts under the same window cut into "
                        "token ranges of every plane (H3_LAUNCH_CHUNK_TOKENS)"}
    if hasattr(step, "close"):
        timer.synchronize()
        barrier(local, timer)
        step.close()
    del step
    return result


# ---------------------------------------------------------------------------
# the oracle on the host cores
# ---------------------------------------------------------------------------

class OracleStep:
    """The step through the CPU oracle on a sample of the workload: `tokens`
    tokens of the relayout problem (same planes, heads and W) and `rows` rows
    of the reduce-scatter (same C and W)."""

    def __init__(self, tokens: int, rows: int):
        import oracle
        self.o = oracle.load()
        rw, red = RELAYOUT, REDUCE
        self.T, self.W, self.P, self.H, self.D = tokens, rw.W, rw.P, rw.H, rw.D
        self.Tr, self.Wr, self.C = rows, red.W, red.C
        self.bounds = wl.segment_bounds(tokens, min(rw.n_segs, tokens), rw.seed)
        full = wl.bf16_bits(wl.normal_bf16((tokens, self.P, self.H, self.D), rw.seed))
        ts = self.o.partition_range(tokens, self.W)
        self.send = [full[ts[r]:ts[r + 1]] for r in range(self.W)]
        w = wl.ReduceWorkload("sample", T=rows, C=self.C, W=self.Wr, seed=red.seed)
        partials, bias = wl.partials_and_bias(w, "cpu")
        self.partials = [wl.bf16_bits(p) for p in partials.unbind(0)]
        self.bias = wl.bf16_bits(bias)
        self.bytes = (2 * relayout_bytes(tokens, self.P, self.H, self.D)
                      + reduce_bytes(rows, self.C, self.Wr))

    def run(self):
        o = self.o
        ts = o.partition_range(self.T, self.W)
        for r in range(self.W):
            o.clip_segments(self.bounds, int(ts[r]), int(ts[r + 1]))
        heads = o.seq_to_head(self.send, self.T, self.P, self.H, self.D, self.W)
        o.head_to_seq(heads, self.T, self.P, self.H, self.D, self.W)
        o.ragged_reduce_scatter(self.partials, self.bias, self.Wr)


def sample_rows(tokens: int) -> int:
    """Reduce-scatter rows that go with `tokens` relayout tokens in a sample,
    so that the sample keeps the step's mix of the two problems."""
    return max(REDUCE.W, round(tokens * REDUCE.T / RELAYOUT.T))


def sample_text(tokens: int) -> str:
    return (f"{tokens} of {RELAYOUT.T} tokens of the QKVG round trip (W={RELAYOUT.W}) and "
            f"{sample_rows(tokens)} of {REDUCE.T} rows of the reduce-scatter (W={REDUCE.W}), "
            f"shapes otherwise the step's")


def oracle_seconds_per_token() -> float:
    s = OracleStep(256, sample_rows(256))
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
    sample per thread, run concurrently (the C oracle is called without the
    GIL, so the threads use separate cores)."""

    def __init__(self, tokens_each: int, threads: int):
        from concurrent.futures import ThreadPoolExecutor
        self.steps = [OracleStep(tokens_each, sample_rows(tokens_each)) for _ in range(threads)]
        self.tokens_each = tokens_each
        self.bytes = sum(s.bytes for s in self.steps)
        self.pool = ThreadPoolExecutor(max_workers=threads)

    def run(self):
        list(self.pool.map(lambda s: s.run(), self.steps))

    def close(self):
        self.pool.shutdown()


# tokens of one thread's sample: bounds host memory (about 210 KB per token)
MAX_TOKENS_PER_THREAD = 1024


def cpu_baseline(budget_s: float = 12.0) -> dict:
    """The oracle on every host core (the reported value) and on one core
    (`one_core`), each on a bounded sample of the bench step."""
    per_tok = oracle_seconds_per_token()
    # one core: the step on one sample, best of 2
    tokens = int(min(RELAYOUT.T, max(RELAYOUT.W, budget_s / 4 / per_tok)))
    s = OracleStep(tokens, sample_rows(tokens))
    times = []
    for _ in range(2):
        t0 = time.perf_counter()
        s.run()
        times.append(time.perf_counter() - t0)
    t1 = min(times)
    one = {"value": round(s.bytes / t1 / 1e9, 3), "unit": UNIT, "cores": 1, "kind": "oracle",
           "sample": f"the step on {sample_text(tokens)}, best of 2, {t1:.2f} s each, "
                     f"single-threaded C oracle"}
    del s
    # every core: one sample per thread, repeated for about budget/2 seconds
    cores = host_cores()
    each = int(max(RELAYOUT.W, min(MAX_TOKENS_PER_THREAD, budget_s / 8 / per_tok)))
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
            "sample": f"{cores} threads, each the step on its own {sample_text(each)}; "
                      f"{n} rounds in {t:.1f} s, C oracle unchanged",
            "cpu_model": host_cpu_model(), "one_core": one}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    budget = float(args.reference_budget)  # seconds for warm-up + timed steps
    per_tok = oracle_seconds_per_token()
    per_step = budget / max(1, args.steps + args.warmup)
    cores = host_cores()
    each = int(min(MAX_TOKENS_PER_THREAD, max(RELAYOUT.W, per_step / per_tok)))
    s = OracleSteps(each, cores)
    for _ in range(args.warmup):
        s.run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        s.run()
    t = time.perf_counter() - t0
    s.close()
    value = s.bytes * args.steps / t / 1e9
    sample = f"each step: {cores} threads, each the path on its own {sample_text(each)}; C oracle unchanged"
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(t / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "accumulate_dtype": "f32",
        "data": "synthetic",
        "config": step_config(world),
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample, "cpu_model": host_cpu_model(),
                         "sample_tokens": each * cores, "sample_rows": sample_rows(each) * cores},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def run_profile(args):
    """Run one kernel of the path --steps times (for ncu captures); no timing.
    The step's kernels (--profile-tokens shrinks the relayout problem,
    --profile-rows the reduce-scatter), and the widened rows on the same
    shapes: gated reduce-scatter (16 segments), all-gather of the reduce
    outputs, staged seq->head through the 896,000,000-byte window, and rank
    0's pulled seq->head share."""
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    relayout = args.profile in ("seq_to_head", "head_to_seq", "staged_seq_to_head", "rank_seq_to_head")
    step = Step(device, tokens=args.profile_tokens, rows=args.profile_rows, relayout=relayout,
                reduce=not relayout)
    if args.profile_window >= 0:
        step.window = args.profile_window
    rr = step.rr
    if args.profile == "head_to_seq":
        rr.seq_to_head(step.send, step.heads)
    extra = {}
    if args.profile == "gated_reduce_scatter":
        extra["bounds"] = wl.segment_bounds(step.Tr, 16, REDUCE.seed)
        extra["gate"] = wl.normal_bf16((16, step.C), REDUCE.seed + 2, 1.0, device)
        extra["x_full"], extra["x"] = rr.alloc_reduce_outputs(step.Tr, step.C, step.Wr, device)
        extra["x_full"].copy_(wl.normal_bf16((step.Tr, step.C), REDUCE.seed + 3, 1.0, device))
    elif args.profile == "all_gather":
        rr.ragged_reduce_scatter(step.partial_list, step.bias, step.red_out)
        extra["outs"] = [torch.empty((step.Tr, step.C), dtype=torch.bfloat16, device=device)
                         for _ in range(step.Wr)]
    elif args.profile == "staged_seq_to_head":
        extra["win"] = torch.empty(WINDOW, dtype=torch.uint8, device=device)
    elif args.profile == "rank_seq_to_head":
        extra["mine"] = torch.empty_like(step.heads[0])
    layout = args.profile_layout
    if layout and args.profile in ("seq_to_head", "head_to_seq"):
        # the same bytes with plane-major buffers on the sides `layout` names
        part = rr.partition(step.T, step.H, step.W)
        if layout & rr.H3_LAYOUT_SEQ_PLANE_MAJOR:
            step.send = [x.permute(1, 0, 2, 3).contiguous() for x in step.send]
            step.back = [torch.empty_like(x) for x in step.send]
        if layout & rr.H3_LAYOUT_HEAD_PLANE_MAJOR:
            step.heads = [torch.empty((step.P, step.T, part.heads(j), step.D), dtype=torch.bfloat16,
                                      device=device) for j in range(step.W)]
        if args.profile == "head_to_seq":
            rr.seq_to_head_layout(step.send, step.heads, layout)
    launches = 0
    for _ in range(args.steps):
        if args.profile == "seq_to_head":
            info = rr.seq_to_head_layout(step.send, step.heads, layout, window_bytes=step.window,
                                         variant=args.profile_variant,
                                         token_chunks=args.profile_token_chunks)
        elif args.profile == "head_to_seq":
            info = rr.head_to_seq_layout(step.heads, step.back, layout, window_bytes=step.window,
                                         variant=args.profile_variant,
                                         token_chunks=args.profile_token_chunks)
        elif args.profile == "reduce_scatter":
            info = rr.ragged_reduce_scatter(step.partial_list, step.bias, step.red_out)
        elif args.profile == "gated_reduce_scatter":
            info = rr.ragged_reduce_scatter_gated(step.partial_list, step.bias, extra["gate"],
                                                  extra["bounds"], extra["x"], step.red_out)
        elif args.profile == "all_gather":
            info = rr.ragged_all_gather(step.red_out, extra["outs"])
        elif args.profile == "staged_seq_to_head":
            info = rr.seq_to_head_staged(step.send, step.heads, extra["win"])
        else:
            info = rr.seq_to_head_rank(step.send, extra["mine"], 0, n_heads=step.H,
                                       window_bytes=step.window)
        launches += info["launches"]
    torch.cuda.synchronize()
    print(json.dumps({"profile": args.profile, "tokens": step.T, "rows": step.Tr,
                      "layout": layout, "window": step.window, "launches": launches,
                      "token_chunks": bool(args.profile_token_chunks)}), flush=True)
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
        if w.T in (32768, 250000):
            # one plane per launch against one launch, with token-major and
            # plane-major buffers (layout bits: 1 sequence side, 2 head side):
            # the cost of one-plane launches on token-major buffers is the
            # interleaving of the planes in memory
            seq_pm = [t.permute(1, 0, 2, 3).contiguous() for t in send]
            heads_pm = [torch.empty((w.P, w.T, part.heads(j), w.D), dtype=torch.bfloat16, device=dev)
                        for j in range(w.W)]
            back_pm = [torch.empty_like(t) for t in seq_pm]
            for layout in (0, 1, 2, 3):
                lsend = seq_pm if layout & 1 else send
                lback = back_pm if layout & 1 else back
                lheads = heads_pm if layout & 2 else heads
                # the same window cut into token ranges of every plane
                # (H3_LAUNCH_CHUNK_TOKENS), on token-major buffers
                shapes = [(0, False, "unchunked"), (WINDOW, False, "chunked")]
                if layout == 0:
                    shapes.append((WINDOW, True, "token_ranges"))
                for wb, tok, kind in shapes:
                    tag = f"layout{layout}_{kind}"
                    info = rr.seq_to_head_layout(lsend, lheads, layout, window_bytes=wb, token_chunks=tok)
                    secs = _time_calls(lambda: rr.seq_to_head_layout(
                        lsend, lheads, layout, window_bytes=wb, token_chunks=tok), iters)
                    emit(w.name, "seq_to_head", tag, nbytes, secs, info)
                    info = rr.head_to_seq_layout(lheads, lback, layout, window_bytes=wb, token_chunks=tok)
                    secs = _time_calls(lambda: rr.head_to_seq_layout(
                        lheads, lback, layout, window_bytes=wb, token_chunks=tok), iters)
                    emit(w.name, "head_to_seq", tag, nbytes, secs, info)
                    if not all(torch.equal(a.view(torch.int16), b.view(torch.int16))
                               for a, b in zip(lback, lsend)):
                        raise SystemExit(f"{w.name} {tag}: round trip differs")
            del seq_pm, heads_pm, back_pm
            torch.cuda.empty_cache()
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
            # the same W shares at once, one stream each: every source row is
            # read by all W pulls at about the same time, as when W GPUs pull
            # from one GPU's memory (no share waits on another)
            side = [torch.cuda.Stream(dev) for _ in range(w.W)]

            def concurrently(share):
                def fn():
                    cur = torch.cuda.current_stream(dev)
                    for st in side:
                        st.wait_stream(cur)
                    for k in range(w.W):
                        last = share(k, side[k])
                    for st in side:
                        cur.wait_stream(st)
                    return last
                return fn

            back_full.zero_()
            for call, fn in (
                    ("seq_to_head", concurrently(lambda k, st: rr.seq_to_head_rank(
                        send, heads[k], k, n_heads=w.H, window_bytes=w.window_bytes, stream=st))),
                    ("head_to_seq", concurrently(lambda k, st: rr.head_to_seq_rank(
                        heads, back[k], k, n_tokens=w.T, window_bytes=w.window_bytes, stream=st)))):
                info = dict(fn())
                info["launches"] *= w.W
                secs = _time_calls(fn, iters)
                emit(w.name, call, "rank_shares_concurrent", nbytes, secs, info)
            torch.cuda.synchronize()
            if not torch.equal(back_full.view(torch.int16), x.view(torch.int16)):
                raise SystemExit(f"{w.name} concurrent rank shares: round trip differs")
            del side
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
    # a plane larger than the window: the long sequence over 2 ranks, where one
    # plane of one rank is 1.79 GB, moves in two token chunks per plane
    w = wl.QKVG_250K_W2_CHUNKED
    x = wl.packed_operand(w, device=dev)
    part = rr.partition(w.T, w.H, w.W)
    send = rr.split_rows(x, part.token_starts)
    heads = rr.alloc_head_side(w.T, w.P, w.H, w.D, w.W, dev)
    back_full, back = rr.alloc_seq_side(w.T, w.P, w.H, w.D, w.W, dev)
    nbytes = 2 * x.numel() * 2
    for wb, tok, tag in ((w.window_bytes, False, "token_chunks"), (w.window_bytes, True, "token_ranges"),
                         (0, False, "unchunked")):
        info = rr.seq_to_head(send, heads, window_bytes=wb, token_chunks=tok)
        secs = _time_calls(lambda: rr.seq_to_head(send, heads, window_bytes=wb, token_chunks=tok), iters)
        emit(w.name, "seq_to_head", tag, nbytes, secs, info)
        info = rr.head_to_seq(heads, back, window_bytes=wb, token_chunks=tok)
        secs = _time_calls(lambda: rr.head_to_seq(heads, back, window_bytes=wb, token_chunks=tok), iters)
        emit(w.name, "head_to_seq", tag, nbytes, secs, info)
        if not torch.equal(back_full.view(torch.int16), x.view(torch.int16)):
            raise SystemExit(f"{w.name} {tag}: round trip differs")
    del x, send, heads, back_full, back
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
        info = rr.ragged_all_gather(blocks, outs, variant=rr.H3_VARIANT_BULK)
        secs = _time_calls(lambda: rr.ragged_all_gather(blocks, outs, variant=rr.H3_VARIANT_BULK), iters)
        emit(f"all_gather_T{T}_C{C_}_W{W}", "ragged_all_gather", "bulk", nbytes, secs, info)
        if not all(torch.equal(o.view(torch.int16), full.view(torch.int16)) for o in outs):
            raise SystemExit("bulk all-gather output differs")
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
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["native", "reference"], default="native")
    p.add_argument("--e2e-steps", type=int, default=10)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-chunk-shapes", action="store_true",
                   help="skip the token-range relayouts timed beside the line (chunk_shapes), "
                        "e.g. for a launch list of the step's own kernels")
    p.add_argument("--cpu-budget", type=float, default=12.0,
                   help="about how many seconds cpu_baseline spends on the oracle")
    p.add_argument("--profile", choices=["seq_to_head", "head_to_seq", "reduce_scatter",
                                         "gated_reduce_scatter", "all_gather",
                                         "staged_seq_to_head", "rank_seq_to_head"],
                   help="run only this kernel of the step --steps times (ncu captures); no timing")
    p.add_argument("--profile-tokens", type=int, default=RELAYOUT.T)
    p.add_argument("--profile-rows", type=int, default=REDUCE.T)
    p.add_argument("--profile-window", type=int, default=-1,
                   help="window bytes of the relayouts for --profile (-1: the bench's 896,000,000; "
                        "0: one launch over all planes)")
    p.add_argument("--profile-variant", type=int, default=0,
                   help="relayout kernel family for --profile: 0 default, 1 vector, 2 bulk (TMA)")
    p.add_argument("--profile-token-chunks", action="store_true",
                   help="relayouts for --profile cut the window into token ranges of every plane "
                        "(H3_LAUNCH_CHUNK_TOKENS) instead of one plane per launch")
    p.add_argument("--profile-layout", type=int, default=0,
                   help="relayout buffers for --profile: bit 1 sequence side plane-major, "
                        "bit 2 head side plane-major (h3_*_layout)")
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
