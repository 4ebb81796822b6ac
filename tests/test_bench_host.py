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


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--gpus", "2", "--steps", "2", "--warmup", "3"],
                         capture_output=True, text=True, env=env, timeout=120)
    assert out.returncode == 0 and out.stdout.strip() == ""
