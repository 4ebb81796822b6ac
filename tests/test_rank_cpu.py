"""Host side of the one-rank-per-GPU calls, on the CPU.

* Argument checks of ``h3_*_rank`` and ``h3_ipc_*``: made-up device addresses
  (never dereferenced) that each fail a host-side check, so nothing is
  launched; run only with no GPU visible.
* ``peers.PeerBuffers`` with two gloo ranks and a fake IPC backend: the
  exchange order, the pointer table and the unmapping.
"""
import ctypes as C
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from ragged_reduce_b200 import _abi, peers

NO_GPU = not torch.cuda.is_available()
needs_no_gpu = pytest.mark.skipif(not NO_GPU, reason="made-up pointers are only passed with no GPU visible")
BASE = 1 << 41
E = _abi


def _split(n, w):
    q, m = divmod(n, w)
    return [i * q + min(i, m) for i in range(w + 1)]


def _seq_head_layout(T, P, H, D, W):
    ts, hs = _split(T, W), _split(H, W)
    addr = BASE
    seq, head = [], []
    for r in range(W):
        seq.append(addr)
        addr += (ts[r + 1] - ts[r]) * P * H * D * 2 + 4096
    for j in range(W):
        head.append(addr)
        addr += T * P * (hs[j + 1] - hs[j]) * D * 2 + 4096
    return seq, head, addr


def _call_relayout(fn, send, recv, T, P, H, D, W, rank, window=0, cfg=None):
    info = _abi.ExecInfo()
    st = getattr(_abi.lib, fn)(_abi.pointer_array(send), C.c_void_p(recv), T, P, H, D, W, rank,
                               window, None, cfg, C.byref(info))
    assert info.launches == 0
    return st


@needs_no_gpu
def test_relayout_rank_argument_checks():
    T, P, H, D, W = 1000, 3, 56, 128, 6
    seq, head, free = _seq_head_layout(T, P, H, D, W)
    for fn, send, recv_of in (("h3_seq_to_head_rank", seq, lambda k: head[k]),
                              ("h3_head_to_seq_rank", head, lambda k: seq[k])):
        # rank out of range, NULL arrays, NULL entries
        for rank in (-1, W, 99):
            assert _call_relayout(fn, send, free, T, P, H, D, W, rank) == E.H3_ERR_INVALID_ARG
        info = _abi.ExecInfo()
        assert getattr(_abi.lib, fn)(None, C.c_void_p(free), T, P, H, D, W, 0, 0, None, None,
                                     C.byref(info)) == E.H3_ERR_INVALID_ARG
        assert _call_relayout(fn, send[:-1] + [0], free, T, P, H, D, W, 0) == E.H3_ERR_INVALID_ARG
        assert _call_relayout(fn, send, 0, T, P, H, D, W, 0) == E.H3_ERR_INVALID_ARG
        # empty partitions, misalignment, too large
        assert _call_relayout(fn, send, free, T, P, H, D, 57, 0) == E.H3_ERR_EMPTY_PARTITION
        assert _call_relayout(fn, send, free + 8, T, P, H, D, W, 0) == E.H3_ERR_MISALIGNED
        assert _call_relayout(fn, [send[0] + 8] + send[1:], free, T, P, H, D, W, 0) == E.H3_ERR_MISALIGNED
        assert _call_relayout(fn, send, free, T, P, H, 4, W, 0) == E.H3_ERR_MISALIGNED
        # the output overlapping any input, the rank's own or a peer's
        for k in range(W):
            assert _call_relayout(fn, send, send[k] + 4096 * 4, T, P, H, D, W, k) == E.H3_ERR_INVALID_ARG
        # a window that cannot hold one token of every rank (6 ranks x 10 heads)
        assert _call_relayout(fn, send, free, T, P, H, D, W, 0, window=6 * 10 * D * 2 - 16) == E.H3_ERR_WINDOW
        assert _call_relayout(fn, send, free, T, P, H, D, W, 0, window=-1) == E.H3_ERR_INVALID_ARG
        # bulk is not offered; unknown variants and flags are rejected
        bulk = C.byref(_abi.LaunchConfig(E.H3_VARIANT_BULK, 0, 0, 0))
        assert _call_relayout(fn, send, free, T, P, H, D, W, 0, cfg=bulk) == E.H3_ERR_UNSUPPORTED
        for cfg in (_abi.LaunchConfig(7, 0, 0, 0), _abi.LaunchConfig(0, -1, 0, 0),
                    _abi.LaunchConfig(0, 0, 4, 0), _abi.LaunchConfig(0, 0, 0, 1)):
            assert _call_relayout(fn, send, free, T, P, H, D, W, 0, cfg=C.byref(cfg)) == E.H3_ERR_INVALID_ARG
        # token-range chunks are a relayout option: the window check applies to
        # one token of every plane (P = 3 planes here)
        tok = C.byref(_abi.LaunchConfig(0, 0, _abi.H3_LAUNCH_CHUNK_TOKENS, 0))
        assert _call_relayout(fn, send, free, T, P, H, D, W, 0, cfg=tok,
                              window=P * 6 * 10 * D * 2 - 16) == E.H3_ERR_WINDOW


@needs_no_gpu
def test_rows_rank_argument_checks():
    T, Cc, W = 1000, 7168, 6
    ts = _split(T, W)
    addr = BASE
    full, blocks = [], []
    for _ in range(W):
        full.append(addr)
        addr += T * Cc * 2 + 4096
    for r in range(W):
        blocks.append(addr)
        addr += (ts[r + 1] - ts[r]) * Cc * 2 + 4096
    bias = addr
    addr += Cc * 2 + 4096
    out = addr

    def rs(parts=full, b=bias, o=out, T=T, Cc=Cc, W=W, rank=0, cfg=None):
        info = _abi.ExecInfo()
        st = _abi.lib.h3_ragged_reduce_scatter_rank(_abi.pointer_array(parts), C.c_void_p(b),
                                                    C.c_void_p(o), T, Cc, W, rank, None, cfg,
                                                    C.byref(info))
        assert info.launches == 0
        return st

    def ag(ins=blocks, o=out, T=T, Cc=Cc, W=W, rank=0, cfg=None):
        info = _abi.ExecInfo()
        st = _abi.lib.h3_ragged_all_gather_rank(_abi.pointer_array(ins), C.c_void_p(o), T, Cc, W,
                                                rank, None, cfg, C.byref(info))
        assert info.launches == 0
        return st

    for f, ins in ((rs, full), (ag, blocks)):
        assert f(rank=-1) == E.H3_ERR_INVALID_ARG
        assert f(rank=W) == E.H3_ERR_INVALID_ARG
        assert f(T=W - 1) == E.H3_ERR_EMPTY_PARTITION
        assert f(W=65) == E.H3_ERR_UNSUPPORTED
        assert f(Cc=7164) == E.H3_ERR_MISALIGNED
        assert f(o=out + 8) == E.H3_ERR_MISALIGNED
        assert f(o=0) == E.H3_ERR_INVALID_ARG
        assert f(o=ins[2] + 4096) == E.H3_ERR_INVALID_ARG      # output inside an input
        assert f(cfg=C.byref(_abi.LaunchConfig(0, 0, 4, 0))) == E.H3_ERR_INVALID_ARG
        # token-range chunks only mean something to the relayouts
        assert f(cfg=C.byref(_abi.LaunchConfig(0, 0, _abi.H3_LAUNCH_CHUNK_TOKENS, 0))) == E.H3_ERR_INVALID_ARG
        if f is rs:
            assert f(parts=full[:-1] + [full[-1] + 8]) == E.H3_ERR_MISALIGNED
        else:
            assert f(ins=blocks[:-1] + [blocks[-1] + 8]) == E.H3_ERR_MISALIGNED
    assert rs(b=bias + 2) == E.H3_ERR_MISALIGNED
    assert rs(o=bias) == E.H3_ERR_INVALID_ARG                     # output over the bias
    assert ag(cfg=C.byref(_abi.LaunchConfig(E.H3_VARIANT_BULK, 0, 0, 0))) == E.H3_ERR_UNSUPPORTED
    assert rs(cfg=C.byref(_abi.LaunchConfig(E.H3_VARIANT_VECTOR, 0, 0, 0))) == E.H3_ERR_INVALID_ARG


@needs_no_gpu
def test_gated_rank_argument_checks():
    T, Cc, W, S = 1000, 1024, 4, 3
    addr = BASE
    parts = []
    for _ in range(W):
        parts.append(addr)
        addr += T * Cc * 2 + 4096
    gate = addr
    addr += S * Cc * 2 + 4096
    x = addr
    addr += T * Cc * 2 + 4096
    bounds = np.array([0, 100, 700, T], dtype=np.int64)

    def st(bounds=bounds, n=S, gate=gate, x=x, out=x, rank=1, bias=0):
        info = _abi.ExecInfo()
        s = _abi.lib.h3_ragged_reduce_scatter_gated_rank(
            _abi.pointer_array(parts), C.c_void_p(bias), C.c_void_p(gate),
            bounds.ctypes.data_as(C.POINTER(C.c_int64)), n, C.c_void_p(x), C.c_void_p(out), T, Cc,
            W, rank, None, None, C.byref(info))
        assert info.launches == 0
        return s

    assert st(n=0) == E.H3_ERR_INVALID_ARG
    assert st(n=257) == E.H3_ERR_UNSUPPORTED
    assert st(bounds=np.array([0, 100, 100, T], dtype=np.int64)) == E.H3_ERR_INVALID_ARG
    assert st(bounds=np.array([1, 100, 700, T], dtype=np.int64)) == E.H3_ERR_INVALID_ARG
    assert st(bounds=np.array([0, 100, 700, T - 1], dtype=np.int64)) == E.H3_ERR_INVALID_ARG
    assert st(gate=gate + 8) == E.H3_ERR_MISALIGNED
    assert st(x=x + 8, out=x + 8) == E.H3_ERR_MISALIGNED
    assert st(out=gate) == E.H3_ERR_INVALID_ARG            # output over the gate rows
    assert st(out=parts[1] + 4096) == E.H3_ERR_INVALID_ARG  # output inside a partial
    assert st(out=x + 16) == E.H3_ERR_INVALID_ARG           # overlapping, not identical, residual
    assert st(rank=W) == E.H3_ERR_INVALID_ARG
    assert st(gate=0) == E.H3_ERR_INVALID_ARG


@needs_no_gpu
def test_gated_rank_checks_at_the_largest_world():
    """W = 64 partials plus gate, residual and bias all reach the overlap
    check (the largest input set a rank call examines)."""
    T, Cc, W, S = 256, 64, 64, 64
    addr = BASE
    parts = []
    for _ in range(W):
        parts.append(addr)
        addr += T * Cc * 2 + 4096
    gate, bias = addr, addr + S * Cc * 2 + 4096
    x = bias + Cc * 2 + 4096
    bounds = np.arange(0, T + 1, T // S, dtype=np.int64)
    for out, want in ((x + 16, E.H3_ERR_INVALID_ARG),      # overlaps the residual
                      (bias, E.H3_ERR_INVALID_ARG),        # over the bias
                      (parts[63] + 64, E.H3_ERR_INVALID_ARG)):
        info = _abi.ExecInfo()
        st = _abi.lib.h3_ragged_reduce_scatter_gated_rank(
            _abi.pointer_array(parts), C.c_void_p(bias), C.c_void_p(gate),
            bounds.ctypes.data_as(C.POINTER(C.c_int64)), S, C.c_void_p(x), C.c_void_p(out), T, Cc,
            W, 63, None, None, C.byref(info))
        assert st == want and info.launches == 0


def test_bounded_wait_selftest_argument_checks():
    out = C.c_int32(7)
    for polls, arrive in ((0, 0), ((1 << 24) + 1, 0), (16, 2), (16, -1)):
        assert _abi.lib.h3_bounded_wait_selftest(polls, arrive, None, C.byref(out)) == E.H3_ERR_INVALID_ARG
    assert out.value == 7  # untouched on an argument error
    assert _abi.lib.h3_bounded_wait_selftest(16, 0, None, None) == E.H3_ERR_INVALID_ARG


def test_ipc_null_and_bad_records():
    h = _abi.IpcHandle()
    ptr = C.c_void_p()
    assert _abi.lib.h3_ipc_export(None, C.byref(h)) == E.H3_ERR_INVALID_ARG
    assert _abi.lib.h3_ipc_open(None, C.byref(ptr)) == E.H3_ERR_INVALID_ARG
    assert _abi.lib.h3_ipc_open(C.byref(h), None) == E.H3_ERR_INVALID_ARG
    h.offset, h.alloc_bytes = 64, 64          # offset past the allocation
    assert _abi.lib.h3_ipc_open(C.byref(h), C.byref(ptr)) == E.H3_ERR_INVALID_ARG
    h.offset = -16
    assert _abi.lib.h3_ipc_open(C.byref(h), C.byref(ptr)) == E.H3_ERR_INVALID_ARG
    assert _abi.lib.h3_ipc_close(None, C.byref(h)) == E.H3_ERR_INVALID_ARG
    assert _abi.lib.h3_ipc_close(C.c_void_p(BASE), C.byref(h)) == E.H3_ERR_INVALID_ARG
    assert C.sizeof(_abi.IpcHandle) == 80


class FakeIpc:
    """Records instead of CUDA calls: rank r's 'handle' names r and its address."""

    def __init__(self, rank):
        self.rank = rank
        self.opened, self.closed = [], []

    def export(self, tensor):
        return b"rank%d:%d" % (self.rank, tensor.data_ptr())

    def open(self, record, device):
        src, addr = record.decode().split(":")
        mapped = (1 << 44) + int(src[4:]) * (1 << 30)   # a distinct made-up mapping per peer
        self.opened.append((src, int(addr)))
        return mapped

    def close(self, address, record, device):
        self.closed.append((address, record))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _peer_worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = torch.zeros(16 + rank, 8, dtype=torch.bfloat16)
        fake = FakeIpc(rank)
        table = peers.PeerBuffers(local, ipc=fake)
        result = (rank, list(table.pointers), table.shapes, fake.opened[:], local.data_ptr())
        table.close()
        out_q.put(result + (fake.closed[:], table.pointers))
    finally:
        dist.destroy_process_group()


def test_peer_buffers_exchange_with_gloo():
    world = 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_peer_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, pointers, shapes, opened, own, closed, after in res:
        assert len(pointers) == world
        assert shapes == [(16 + r, 8) for r in range(world)]
        for r in range(world):
            if r == rank:
                assert pointers[r] == own
            else:
                assert pointers[r] == (1 << 44) + r * (1 << 30)
        assert sorted(s for s, _ in opened) == sorted(f"rank{r}" for r in range(world) if r != rank)
        assert sorted(a for a, _ in closed) == sorted(p for r, p in enumerate(pointers) if r != rank)
        assert after == []


def test_rank_reduce_wrappers_require_bf16():
    """The reduce arithmetic reads BF16: a tensor of another 2-byte type is
    refused by the binding; raw device addresses carry no type."""
    import ragged_reduce_b200 as rr
    rr._require_bf16([torch.zeros(4, dtype=torch.bfloat16), 0x10000, None], "ok")
    for dt in (torch.float16, torch.int16):
        with pytest.raises(ValueError, match="BF16"):
            rr._require_bf16([torch.zeros(4, dtype=torch.bfloat16), torch.zeros(4, dtype=dt)], "bad")
