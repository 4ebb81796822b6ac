"""bench.py with one rank per GPU, on the CPU: the host logic of the sharded
step with two and three gloo ranks.

Every process runs ``bench.measure`` on a ``bench.ShardedStep`` exactly as
``bench.py --gpus N`` does under torchrun, with three stand-ins for what needs
GPUs:

* the buffers the peers read live in shared files mapped by every process
  (``ShmIpc``), so that one rank's writes are seen by the others;
* the rank calls are torch restatements of the library's rank shares on CPU
  tensors (``FakeRankCalls``), resolving the pointer tables through the
  mappings; ``partition`` is the library's own host call;
* the fence between calls is a gloo all-reduce.

Checked: the line rank 0 prints (parallelism names the rank split, strong
scaling, whole-job bytes, every kernel timed, launches summed over ranks),
the order of the calls and fences in every step, the peer tables' exchange
order, and that the per-rank check of the results catches a wrong share.
"""
import json
import os
import socket
import sys
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import ragged_reduce_b200 as rr  # noqa: E402
from ragged_reduce_b200 import peers  # noqa: E402

TOKENS, ROWS = 90, 40


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class ShmIpc:
    """Buffers in shared files: allocation, export, mapping and the address
    registry the fake rank calls resolve pointers with."""

    def __init__(self, folder, rank):
        self.folder, self.rank, self.n = folder, rank, 0
        self.by_address = {}
        self.files = {}
        self.opened, self.closed = [], []

    def empty(self, shape, dtype):
        numel = int(np.prod(shape))
        path = os.path.join(self.folder, f"r{self.rank}_{self.n}.bin")
        self.n += 1
        with open(path, "wb") as f:
            f.truncate(numel * torch.empty((), dtype=dtype).element_size())
        t = torch.from_file(path, shared=True, size=numel, dtype=dtype).view(shape)
        self.by_address[t.data_ptr()] = t
        self.files[t.data_ptr()] = (path, tuple(shape), str(dtype))
        return t

    def export(self, tensor):
        path, shape, dtype = self.files[tensor.data_ptr()]
        return json.dumps([path, list(shape), dtype]).encode()

    def open(self, record, device):
        path, shape, dtype = json.loads(record.decode())
        dt = getattr(torch, dtype.split(".")[1])
        t = torch.from_file(path, shared=True, size=int(np.prod(shape)), dtype=dt).view(shape)
        self.by_address[t.data_ptr()] = t
        self.opened.append(os.path.basename(path))
        return t.data_ptr()

    def close(self, address, record, device):
        self.closed.append(address)


class FakeRankCalls:
    """The library's rank shares restated with torch on CPU tensors."""

    def __init__(self, ipc, log, corrupt=False):
        self.ipc, self.log, self.corrupt = ipc, log, corrupt

    partition = staticmethod(rr.partition)

    def _t(self, address):
        return self.ipc.by_address[int(address)]

    def seq_to_head_rank(self, send, recv, k, *, n_heads, window_bytes=0, stream=None):
        W = len(send)
        T, P = recv.shape[0], recv.shape[1]
        part = rr.partition(T, n_heads, W)
        hs, he = int(part.head_starts[k]), int(part.head_starts[k + 1])
        for r in range(W):
            ts, te = int(part.token_starts[r]), int(part.token_starts[r + 1])
            recv[ts:te] = self._t(send[r])[:, :, hs:he]
        if self.corrupt and k == 0:
            recv[0, 0, 0, 0] += 1
        self.log.append(("seq_to_head", k, window_bytes))
        return {"launches": P if window_bytes else 1}

    def head_to_seq_rank(self, send, recv, k, *, n_tokens, window_bytes=0, stream=None):
        W = len(send)
        H, P = recv.shape[2], recv.shape[1]
        part = rr.partition(n_tokens, H, W)
        ts, te = int(part.token_starts[k]), int(part.token_starts[k + 1])
        for j in range(W):
            hs, he = int(part.head_starts[j]), int(part.head_starts[j + 1])
            recv[:, :, hs:he] = self._t(send[j])[ts:te]
        self.log.append(("head_to_seq", k, window_bytes))
        return {"launches": P if window_bytes else 1}

    def ragged_reduce_scatter_rank(self, partials, bias, out, k, *, n_tokens, stream=None):
        W = len(partials)
        part = rr.partition(n_tokens, W, W)
        ts, te = int(part.token_starts[k]), int(part.token_starts[k + 1])
        acc = self._t(partials[0])[ts:te].float()
        for r in range(1, W):
            acc += self._t(partials[r])[ts:te].float()
        acc += bias.float()
        out.copy_(acc.to(torch.bfloat16))
        self.log.append(("reduce_scatter", k))
        return {"launches": 1}


def _worker(rank, world, port, folder, corrupt, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ipc = ShmIpc(folder, rank)
        log = []
        fake = FakeRankCalls(ipc, log, corrupt=corrupt)
        token = torch.zeros(1)

        def fence(stream=None):
            log.append(("fence",))
            dist.all_reduce(token)

        def table(t):
            log.append(("table", tuple(t.shape)))
            return peers.PeerBuffers(t, ipc=ipc)

        def make_step():
            return bench.ShardedStep("cpu", rank, world, rr=fake, peer_table=table, fence=fence,
                                     tokens=TOKENS, rows=ROWS, empty=ipc.empty)

        args = bench.parse_args(["--gpus", str(world), "--steps", "3", "--warmup", "3"])
        try:
            result = bench.measure(args, make_step, rank, world, rank, "cpu", bench.HostTimer(), 5)
            out_q.put((rank, "ok", result, log, ipc.opened, ipc.closed))
        except SystemExit as e:
            out_q.put((rank, "exit", str(e), log, ipc.opened, ipc.closed))
    finally:
        dist.destroy_process_group()


def _run(world, corrupt=False):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    with tempfile.TemporaryDirectory() as folder:
        procs = [ctx.Process(target=_worker, args=(r, world, port, folder, corrupt, q))
                 for r in range(world)]
        for p in procs:
            p.start()
        res = sorted((q.get(timeout=300) for _ in procs), key=lambda x: x[0])
        for p in procs:
            p.join(timeout=60)
            assert p.exitcode == 0
    return res


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_bench_line_and_call_order(world):
    res = _run(world)
    assert [r[1] for r in res] == ["ok"] * world, res
    line = res[0][2]
    assert all(r[2] is None for r in res[1:])            # only rank 0 prints
    assert line["n_gpus"] == world and line["scaling"] == "strong"
    assert f"W={world}" in line["config"]["parallelism"]
    assert "one rank per GPU" in line["config"]["parallelism"]
    assert line["config"]["workload"] == bench.WORKLOAD
    assert line["config"]["relayout"]["world"] == world
    H, D, P, C = 56, 128, bench.RELAYOUT.P, bench.REDUCE.C
    want = (2 * bench.relayout_bytes(TOKENS, P, H, D) + bench.reduce_bytes(ROWS, C, world)
            + (world - 1) * C * 2)
    assert line["config"]["bytes_per_step"] == want
    assert set(line["kernels"]) == set(bench.KERNELS)
    # launches: per rank and step 4 planes each way (one batch plane per
    # launch) and one reduce launch, summed over ranks
    assert line["gpu_launches"] == world * 3 * (P + P + 1)
    assert line["roofline"]["traffic"] is None
    assert set(line["nvlink_rank0"]) == set(bench.KERNELS)
    for rank, _, _, log, opened, closed in res:
        # the tables, in the same order on every rank: sequence side, head side, partial
        tables = [e for e in log if e[0] == "table"]
        assert [len(e[1]) for e in tables] == [4, 4, 2]
        assert len(opened) == 3 * (world - 1) and len(closed) == len(opened)
        # every step: seq->head, fence, head->seq, reduce-scatter, fence
        calls = [e for e in log if e[0] != "table"]
        steps = 3 + 3                                    # warm-up + timed
        assert len(calls) == steps * 5
        for s in range(steps):
            chunk = calls[5 * s: 5 * s + 5]
            assert [c[0] for c in chunk] == ["seq_to_head", "fence", "head_to_seq",
                                             "reduce_scatter", "fence"]
            assert chunk[0] == ("seq_to_head", rank, bench.WINDOW)
            assert chunk[2] == ("head_to_seq", rank, bench.WINDOW)


def test_sharded_bench_check_catches_a_wrong_share():
    res = _run(2, corrupt=True)
    assert all(r[1] == "exit" and "wrong results" in r[2] for r in res), res
