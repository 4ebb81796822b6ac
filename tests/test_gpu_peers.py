"""The one-rank-per-GPU path across processes: two or three ranks as
processes sharing one GPU, each holding only its own inputs and mapping the other's
through CUDA IPC (tests/peers_worker.py).  The processes never wait on each
other inside a kernel; gloo barriers order reads after writes.  Checks
seq->head, head->seq, reduce-scatter, gated reduce-scatter and all-gather
against the one-GPU definitions, bit for bit."""
import json
import os
import socket
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WORKER = os.path.join(ROOT, "tests", "peers_worker.py")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3])
def test_processes_pull_from_each_other(world):
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
            out, _ = p.communicate(timeout=300)
            outputs.append(out)
    finally:
        for p in procs:
            if p.poll() is None:
                p.kill()
                p.wait()
    for rank, (p, out) in enumerate(zip(procs, outputs)):
        assert p.returncode == 0, f"rank {rank} exited {p.returncode}:\n{out[-3000:]}"
        line = [l for l in out.splitlines() if l.startswith("{")][-1]
        res = json.loads(line)
        assert res["ok"] and res["rank"] == rank, res
