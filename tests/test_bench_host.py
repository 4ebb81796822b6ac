"""Host logic of bench.py on the CPU: max-over-ranks timing and the whole-job
throughput with two gloo ranks, and the reference arm's JSON line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_time = 1.0 + rank  # rank 1 is the slow one
        t = bench.max_over_ranks(my_time, "cpu")
        launches = bench.sum_over_ranks(5 * (rank + 1), "cpu")
        value = bench.throughput_gbs(1e9, 10, world, t)
        out_q.put((rank, t, launches, value, bench.dist_env()))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_throughput():
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
    for rank, t, launches, value, env in res:
        assert t == 2.0                      # the slowest rank's time
        assert launches == 15                # 5 + 10 launches over both ranks
        assert value == pytest.approx(1e9 * 10 * 2 / 2.0 / 1e9)
        assert env == (rank, 2, rank)


def test_single_process_helpers():
    assert bench.max_over_ranks(3.5, "cpu") == 3.5
    assert bench.throughput_gbs(2e9, 5, 1, 1.0) == pytest.approx(10.0)
    peak, kind = bench.load_peak()
    assert peak > 1000 and kind in ("measured", "fallback")


def test_reference_arm_prints_one_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "2", "--warmup", "3", "--reference-budget", "2"],
                         capture_output=True, text=True, env=env, timeout=300)
    assert out.returncode == 0, out.stderr
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["unit"] == "GB/s" and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
    assert rec["cpu_baseline"]["cpu_model"] == bench.host_cpu_model()
    assert rec["metric"] == bench.METRIC
    # the native arm's config, so that the two lines describe the same workload
    assert rec["config"] == bench.step_config(1)
    assert rec["config"]["bytes_per_step"] == 2 * 2 * 14_336_000_000 + 8_455_731_200


def test_step_config_per_world():
    """The config both arms print: one GPU with 4 (relayout) and 8
    (reduce-scatter) virtual ranks, or N ranks, one per GPU, whose bytes count
    every rank's read of the bias."""
    one = bench.step_config(1)
    assert one["relayout"]["world"] == 4 and one["reduce_scatter"]["world"] == 8
    assert one["relayout"]["chunking"] == "one batch plane per launch"
    for n in (2, 4, 8):
        c = bench.step_config(n)
        assert c["relayout"]["world"] == n and c["reduce_scatter"]["world"] == n
        assert c["bytes_per_step"] == (2 * 2 * 14_336_000_000 + (n + 1) * 65536 * 7168 * 2
                                       + n * 7168 * 2)


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--gpus", "2", "--steps", "2", "--warmup", "3"],
                         capture_output=True, text=True, env=env, timeout=120)
    assert out.returncode == 0 and out.stdout.strip() == ""


def test_traffic_reported_only_for_the_captured_sources(monkeypatch):
    """ncu traffic from profiles/dram_traffic.json is reported while the
    kernel's sources still match the digest recorded with the capture, and
    is None once they differ or the kernel is unknown."""
    entries = json.load(open(os.path.join(ROOT, "profiles", "dram_traffic.json")))
    for kernel in bench.KERNEL_SOURCES:
        e = entries[kernel]
        assert e["bytes_per_launch"] == e["read_bytes"] + e["write_bytes"]
        if e["source_digest"] == bench.kernel_source_digest(kernel):
            assert bench.load_traffic(kernel) == e["bytes_per_launch"]
    assert bench.load_traffic("no_such_kernel") is None
    monkeypatch.setattr(bench, "kernel_source_digest", lambda kernel: "0" * 16)
    for kernel in bench.KERNEL_SOURCES:
        assert bench.load_traffic(kernel) is None


def test_clock_summary():
    """The clock record: median SM clock over the samples, the largest max
    clock, and every throttle reason seen active at least once; malformed
    lines are skipped and no samples give an empty record."""
    c = bench.ClockSampler(None)
    assert c.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
    c.lines = [
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1710, 1965, 998.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1800, 1965, 990.5, 0x4, Not Active, Not Active, Not Active, Active",
        "garbled line",
        "0, [N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    r = c.summary()
    assert r == {"sm_mhz": 1800.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    c.lines.append("0, 1500, 1965, 1000.0, 0x48, Active, Not Active, Active, Active")
    assert c.summary()["reasons"] == ["hw_slowdown", "sw_power_cap", "sw_thermal_slowdown"]
