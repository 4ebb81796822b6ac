"""bench.py's one-rank-per-GPU step on real GPU memory: two and three ranks
as processes sharing one GPU (tests/bench_sharded_worker.py), each holding
only its own buffers and mapping the others' over CUDA IPC.  The warm-up
steps end in each rank's own check of its round trip and reduce rows (the
bench exits on a mismatch); rank 0's line must name the rank split, count
every rank's launches, and carry the end-to-end figures of all ranks."""
import json
import os
import socket
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
WORKER = os.path.join(ROOT, "tests", "bench_sharded_worker.py")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_bench_on_one_gpu(world):
    import bench
    port = _free_port()
    procs = []
    for rank in range(world):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK="0",
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, WORKER], env=env, cwd=ROOT,
                                      stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True))
    outputs = []
    try:
        for p in procs:
            out, _ = p.communicate(timeout=600)
            outputs.append(out)
    finally:
        for p in procs:
            if p.poll() is None:
                p.kill()
                p.wait()
    for rank, (p, out) in enumerate(zip(procs, outputs)):
        assert p.returncode == 0, f"rank {rank} exited {p.returncode}:\n{out[-3000:]}"
    line = json.loads([l for l in outputs[0].splitlines() if l.startswith("{")][-1])
    assert line["n_gpus"] == world and line["scaling"] == "strong"
    assert f"W={world}" in line["config"]["parallelism"]
    P = bench.RELAYOUT.P
    # 3001 tokens: one plane per launch each way, one reduce launch, 5 timed steps per rank
    assert line["gpu_launches"] == world * 5 * (P + P + 1)
    assert set(line["kernels"]) == set(bench.KERNELS) and line["value"] > 0
    e = line["e2e"]
    assert e["round_trip_ok"] is True and e["value"] > 0
    H, D, C = 56, 128, 7168
    # every rank copies in its rows, its partial and the bias; out its rows back and its reduce rows
    assert e["h2d_bytes_per_step"] == 3001 * P * H * D * 2 + world * 1000 * C * 2 + world * C * 2
    assert e["d2h_bytes_per_step"] == 3001 * P * H * D * 2 + 1000 * C * 2
    assert set(line["nvlink_rank0"]) == set(bench.KERNELS)
