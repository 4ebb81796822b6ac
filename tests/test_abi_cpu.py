"""The C-ABI library on the host: exports, the partition plan, argument checks.

No compute call reaches a GPU here.  Tests that pass made-up device pointers
run only when no CUDA device is visible, and each of them is built to fail a
host-side check, so nothing is ever launched.
"""
import ctypes as C
import re

import numpy as np
import pytest
import torch

import ragged_reduce_b200 as rr
from ragged_reduce_b200 import _abi

NO_GPU = not torch.cuda.is_available()


def _declared_functions():
    text = open(_abi.HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"H3RR_API\s+[\w\s\*]+?\b(h3_\w+)\s*\(", text)))


def test_header_declares_the_four_calls():
    names = _declared_functions()
    for n in ("h3_partition", "h3_seq_to_head", "h3_head_to_seq", "h3_ragged_reduce_scatter"):
        assert n in names
    assert len(names) >= 9


def test_library_exports_every_declared_symbol():
    lib = C.CDLL(_abi.LIB_PATH)
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert _abi.lib.h3_abi_version() == _abi.ABI_VERSION


def test_status_strings():
    for code in range(7):
        assert _abi.describe(code) != "unknown status"
    assert _abi.describe(99) == "unknown status"


# ---------------------------------------------------------------------------
# the host plan against the oracle
# ---------------------------------------------------------------------------

def test_partition_head_table(oracle_lib):
    for W, sizes in {2: [28] * 2, 4: [14] * 4, 6: [10, 10, 9, 9, 9, 9], 8: [7] * 8}.items():
        p = rr.partition(1024, 56, W)
        assert list(np.diff(p.head_starts)) == sizes
        assert np.array_equal(p.head_starts, oracle_lib.partition_range(56, W))


def test_partition_matches_oracle_random(oracle_lib):
    rng = np.random.default_rng(21)
    for _ in range(300):
        T = int(rng.integers(1, 300_000))
        W = int(rng.integers(1, 65))
        H = int(rng.integers(W, 200))
        if T < W:
            continue
        S = int(rng.integers(1, min(T, 40) + 1))
        cuts = np.sort(rng.choice(np.arange(1, T), size=S - 1, replace=False)) if S > 1 else []
        bounds = np.concatenate([[0], cuts, [T]]).astype(np.int64)
        p = rr.partition(T, H, W, bounds)
        assert np.array_equal(p.token_starts, oracle_lib.partition_range(T, W))
        assert np.array_equal(p.head_starts.astype(np.int64), oracle_lib.partition_range(H, W))
        for r in range(W):
            lb, ids = oracle_lib.clip_segments(bounds, int(p.token_starts[r]),
                                               int(p.token_starts[r + 1]))
            assert np.array_equal(p.local_bounds[r], lb), (T, W, r)
            assert np.array_equal(p.seg_ids[r], ids), (T, W, r)


def test_partition_tiny_workload_worked_example():
    p = rr.partition(1024, 56, 2, [0, 400, 737, 1024])
    assert list(p.token_starts) == [0, 512, 1024]
    assert [list(b) for b in p.local_bounds] == [[0, 400, 512], [0, 225, 512]]
    assert [list(s) for s in p.seg_ids] == [[0, 1], [1, 2]]


def test_partition_workload_token_starts():
    # quotient/remainder token ranges of the full-size workloads
    assert list(rr.partition(32768, 56, 6).token_starts) == [0, 5462, 10924, 16385, 21846, 27307, 32768]
    assert list(rr.partition(131072, 56, 4).token_starts) == [0, 32768, 65536, 98304, 131072]
    assert list(rr.partition(65536, 56, 8).token_starts) == list(range(0, 65537, 8192))
    assert list(rr.partition(250000, 56, 4).token_starts) == [0, 62500, 125000, 187500, 250000]


@pytest.mark.parametrize("T,H,W,status", [
    (10, 56, 0, _abi.H3_ERR_INVALID_ARG),
    (10, 56, -1, _abi.H3_ERR_INVALID_ARG),
    (10, 5, 6, _abi.H3_ERR_EMPTY_PARTITION),
    (5, 56, 6, _abi.H3_ERR_EMPTY_PARTITION),
    (0, 56, 1, _abi.H3_ERR_EMPTY_PARTITION),
    (1000, 100, 65, _abi.H3_ERR_UNSUPPORTED),
])
def test_partition_rejects(T, H, W, status):
    with pytest.raises(rr.H3Error) as e:
        rr.partition(T, H, W)
    assert e.value.status == status


@pytest.mark.parametrize("bounds", [[0, 5, 5, 10], [1, 5, 10], [0, 5, 9], [0, 7, 3, 10]])
def test_partition_rejects_bad_segments(bounds):
    with pytest.raises(rr.H3Error) as e:
        rr.partition(10, 56, 2, bounds)
    assert e.value.status == _abi.H3_ERR_INVALID_ARG


# ---------------------------------------------------------------------------
# argument checks of the device calls (host only; nothing may launch)
# ---------------------------------------------------------------------------

BASE = 1 << 40  # made-up, never dereferenced


def _ptrs(addrs):
    return _abi.pointer_array(addrs)


def _relayout_status(send, recv, T, P, H, D, W, window=0, fn="h3_seq_to_head"):
    info = _abi.ExecInfo()
    st = getattr(_abi.lib, fn)(_ptrs(send), _ptrs(recv), T, P, H, D, W, window, None,
                               C.byref(info))
    return st, info


def _layout(T, P, H, D, W):
    """Disjoint made-up addresses for send (seq side) and recv (head side)."""
    ts = np.array([r * (T // W) + min(r, T % W) for r in range(W + 1)])
    hs = np.array([j * (H // W) + min(j, H % W) for j in range(W + 1)])
    addr = BASE
    send, recv = [], []
    for r in range(W):
        send.append(addr)
        addr += int(ts[r + 1] - ts[r]) * P * H * D * 2 + 4096
    for j in range(W):
        recv.append(addr)
        addr += T * P * int(hs[j + 1] - hs[j]) * D * 2 + 4096
    return send, recv


needs_no_gpu = pytest.mark.skipif(not NO_GPU, reason="made-up pointers are only passed with no GPU visible")


@needs_no_gpu
@pytest.mark.parametrize("fn", ["h3_seq_to_head", "h3_head_to_seq"])
def test_relayout_argument_checks(fn):
    T, P, H, D, W = 1000, 3, 56, 128, 6
    send, recv = _layout(T, P, H, D, W)
    if fn == "h3_head_to_seq":
        send, recv = recv, send
    E = _abi
    assert _relayout_status(send, recv, T, P, H, D, 0, fn=fn)[0] == E.H3_ERR_INVALID_ARG
    assert _relayout_status(send, recv, T, P, H, D, 65, fn=fn)[0] == E.H3_ERR_UNSUPPORTED
    assert _relayout_status(send[:5] + [send[5]], recv, 5, P, H, D, 6, fn=fn)[0] == E.H3_ERR_EMPTY_PARTITION
    assert _relayout_status(send, recv, T, P, 5, D, 6, fn=fn)[0] == E.H3_ERR_EMPTY_PARTITION
    assert _relayout_status(send, recv, T, 0, H, D, W, fn=fn)[0] == E.H3_ERR_INVALID_ARG
    assert _relayout_status(send, recv, T, P, H, 0, W, fn=fn)[0] == E.H3_ERR_INVALID_ARG
    assert _relayout_status(send, recv, T, P, H, 100, W, fn=fn)[0] == E.H3_ERR_MISALIGNED
    assert _relayout_status(send, recv, T, P, H, D, W, window=-1, fn=fn)[0] == E.H3_ERR_INVALID_ARG
    bad = list(send)
    bad[3] += 8
    assert _relayout_status(bad, recv, T, P, H, D, W, fn=fn)[0] == E.H3_ERR_MISALIGNED
    bad = list(recv)
    bad[5] += 2
    assert _relayout_status(send, bad, T, P, H, D, W, fn=fn)[0] == E.H3_ERR_MISALIGNED
    bad = list(send)
    bad[2] = 0
    assert _relayout_status(bad, recv, T, P, H, D, W, fn=fn)[0] == E.H3_ERR_INVALID_ARG
    # an output overlapping an input, and two outputs overlapping each other
    bad = list(recv)
    bad[1] = send[4] + 1024
    assert _relayout_status(send, bad, T, P, H, D, W, fn=fn)[0] == E.H3_ERR_INVALID_ARG
    bad = list(recv)
    bad[2] = recv[1] + 512
    assert _relayout_status(send, bad, T, P, H, D, W, fn=fn)[0] == E.H3_ERR_INVALID_ARG
    # a window that cannot hold one token of every rank: each head rank
    # receives one token from each of the 6 ranks, 6 x 10 heads x 256 B
    assert _relayout_status(send, recv, T, P, H, D, W, window=6 * 10 * 256 - 1, fn=fn)[0] == E.H3_ERR_WINDOW
    # sizes beyond the kernels' 32-bit row index
    assert _relayout_status(send, recv, 2**31, P, H, D, W, fn=fn)[0] == E.H3_ERR_UNSUPPORTED
    # a NULL pointer array
    info = _abi.ExecInfo()
    assert getattr(_abi.lib, fn)(None, _ptrs(recv), T, P, H, D, W, 0, None, C.byref(info)) == E.H3_ERR_INVALID_ARG
    assert info.launches == 0


@needs_no_gpu
def test_relayout_rejects_unknown_variant():
    T, P, H, D, W = 100, 3, 56, 128, 2
    send, recv = _layout(T, P, H, D, W)
    for variant in (3, 4, 99, -1):
        cfg = _abi.LaunchConfig(variant, 0, 0, 0)
        info = _abi.ExecInfo()
        st = _abi.lib.h3_seq_to_head_ex(_ptrs(send), _ptrs(recv), T, P, H, D, W, 0, None,
                                        C.byref(cfg), C.byref(info))
        assert st == _abi.H3_ERR_INVALID_ARG and info.launches == 0
    cfg = _abi.LaunchConfig(0, -2, 0, 0)
    st = _abi.lib.h3_head_to_seq_ex(_ptrs(recv), _ptrs(send), T, P, H, D, W, 0, None,
                                    C.byref(cfg), C.byref(_abi.ExecInfo()))
    assert st == _abi.H3_ERR_INVALID_ARG


@needs_no_gpu
def test_launch_config_rejects_unknown_flags_and_reserved():
    """H3_LAUNCH_SERIAL is a flag of every _ex call, H3_LAUNCH_CHUNK_TOKENS of
    the relayouts only; reserved1 must be 0."""
    T, P, H, D, W = 100, 3, 56, 128, 2
    send, recv = _layout(T, P, H, D, W)
    Cc = 64
    blocks = [BASE + r * (1 << 20) for r in range(W)]
    full = [BASE + (8 << 20) + r * (1 << 20) for r in range(W)]
    tok = _abi.H3_LAUNCH_CHUNK_TOKENS
    for flags, reserved in ((tok, 0), (tok | _abi.H3_LAUNCH_SERIAL, 0)):
        cfg = C.byref(_abi.LaunchConfig(0, 0, flags, reserved))
        st = _abi.lib.h3_ragged_reduce_scatter_ex(_ptrs(full), None, _ptrs(blocks), T, Cc, W, None,
                                                  cfg, C.byref(_abi.ExecInfo()))
        assert st == _abi.H3_ERR_INVALID_ARG, flags
        st = _abi.lib.h3_ragged_all_gather_ex(_ptrs(blocks), _ptrs(full), T, Cc, W, None, cfg,
                                              C.byref(_abi.ExecInfo()))
        assert st == _abi.H3_ERR_INVALID_ARG, flags
    for flags, reserved in ((4, 0), (-1, 0), (_abi.H3_LAUNCH_SERIAL | 8, 0), (tok | 16, 0), (0, 1),
                            (_abi.H3_LAUNCH_SERIAL, -1), (tok, 1)):
        cfg = C.byref(_abi.LaunchConfig(0, 0, flags, reserved))
        for fn in ("h3_seq_to_head_ex", "h3_head_to_seq_ex"):
            info = _abi.ExecInfo()
            st = getattr(_abi.lib, fn)(_ptrs(send), _ptrs(recv), T, P, H, D, W, 0, None, cfg,
                                       C.byref(info))
            assert st == _abi.H3_ERR_INVALID_ARG and info.launches == 0, (fn, flags, reserved)
        for fn in ("h3_seq_to_head_layout", "h3_head_to_seq_layout"):
            st = getattr(_abi.lib, fn)(_ptrs(send), _ptrs(recv), T, P, H, D, W, 0, 0, None, cfg,
                                       C.byref(_abi.ExecInfo()))
            assert st == _abi.H3_ERR_INVALID_ARG, (fn, flags, reserved)
        st = _abi.lib.h3_ragged_reduce_scatter_ex(_ptrs(full), None, _ptrs(blocks), T, Cc, W, None,
                                                  cfg, C.byref(_abi.ExecInfo()))
        assert st == _abi.H3_ERR_INVALID_ARG, (flags, reserved)
        st = _abi.lib.h3_ragged_all_gather_ex(_ptrs(blocks), _ptrs(full), T, Cc, W, None, cfg,
                                              C.byref(_abi.ExecInfo()))
        assert st == _abi.H3_ERR_INVALID_ARG, (flags, reserved)


def test_bulk_timeout_query_needs_count():
    assert _abi.lib.h3_bulk_wait_timeouts(None, None, 0) == _abi.H3_ERR_INVALID_ARG


@needs_no_gpu
def test_relayout_window_check_long_workload():
    # 250k tokens over 4 ranks: one plane of one rank is exactly 896,000,000
    # bytes, so the pages' window moves one plane per launch; 16 bytes less
    # splits every plane into two token chunks; a window below one token of
    # every rank is refused before anything is launched.
    T, P, H, D, W = 250000, 4, 56, 128, 4
    send, recv = _layout(T, P, H, D, W)
    assert 62500 * 56 * 128 * 2 == 896_000_000
    assert 250000 * 14 * 128 * 2 == 896_000_000
    assert rr.relayout_chunk_plan(T, P, H, D, W, 896_000_000) == (62500, 4)
    assert rr.relayout_chunk_plan(T, P, H, D, W, 896_000_000 - 16) == (31250, 8)
    st, info = _relayout_status(send, recv, T, P, H, D, W, window=H * D * 2 - 16)
    assert st == _abi.H3_ERR_WINDOW and info.launches == 0


def _expected_plan(T, P, H, D, W, window):
    """The chunk plan restated from its definition: one plane per chunk if a
    whole plane of every rank fits; else the fewest token chunks k, and the
    equal length L = ceil(T_max / k), whose full chunks fit."""
    tmax = -(-T // W)
    hmax = -(-H // W)
    row, head = H * D * 2, D * 2
    if tmax * row <= window and T * hmax * head <= window:
        return tmax, P
    for k in range(2, tmax + 1):
        L = -(-tmax // k)
        if L * row <= window and W * L * hmax * head <= window:
            return L, P * k
    return None


def test_relayout_chunk_plan_properties():
    """Against the plan's definition over a grid of shapes and windows, and
    the properties the kernels rely on: full chunks within the window, the
    chunks cover every rank's tokens once, and the last chunk is not empty."""
    rng = np.random.default_rng(5)
    cases = [(250000, 4, 56, 128, 4), (250000, 4, 56, 128, 2), (32768, 3, 56, 128, 6),
             (1000, 3, 56, 128, 8), (777, 1, 7, 64, 3), (64, 2, 56, 128, 56)]
    for _ in range(60):
        W = int(rng.integers(1, 9))
        cases.append((int(rng.integers(W, 5000)), int(rng.integers(1, 5)),
                      int(rng.integers(W, 80)), 8 * int(rng.integers(1, 40)), W))
    for T, P, H, D, W in cases:
        tmax, hmax = -(-T // W), -(-H // W)
        row, head = H * D * 2, D * 2
        smallest = max(row, W * hmax * head)
        windows = {smallest, smallest + 16, T * row, tmax * row, tmax * row - 16,
                   int(rng.integers(smallest, 4 * tmax * row + 1))}
        for win in sorted(windows):
            want = _expected_plan(T, P, H, D, W, win)
            assert want is not None, (T, P, H, D, W, win)
            L, chunks = rr.relayout_chunk_plan(T, P, H, D, W, win)
            assert (L, chunks) == want, (T, P, H, D, W, win)
            k = chunks // P
            if k > 1:
                assert L * row <= win and W * L * hmax * head <= win
                assert (k - 1) * L < tmax <= k * L       # exact cover, last chunk not empty
                # the plan is also the fewest chunks: one fewer would not fit
                Lfew = -(-tmax // (k - 1))
                assert Lfew * row > win or W * Lfew * hmax * head > win
        assert rr.relayout_chunk_plan(T, P, H, D, W, 0) == (tmax, 1)
        with pytest.raises(rr.H3Error) as e:
            rr.relayout_chunk_plan(T, P, H, D, W, smallest - 1)
        assert e.value.status == _abi.H3_ERR_WINDOW


@needs_no_gpu
def test_reduce_argument_checks():
    T, Cc, W = 1000, 7168, 6
    addr = BASE
    parts, outs = [], []
    for _ in range(W):
        parts.append(addr)
        addr += T * Cc * 2 + 4096
    bias = addr
    addr += Cc * 2 + 4096
    for r in range(W):
        outs.append(addr)
        addr += (T // W + 1) * Cc * 2 + 4096

    def st(parts=parts, bias=bias, outs=outs, T=T, Cc=Cc, W=W):
        info = _abi.ExecInfo()
        s = _abi.lib.h3_ragged_reduce_scatter(_ptrs(parts), C.c_void_p(bias), _ptrs(outs), T, Cc,
                                              W, None, C.byref(info))
        assert info.launches == 0
        return s

    E = _abi
    assert st(W=0) == E.H3_ERR_INVALID_ARG
    assert st(W=65) == E.H3_ERR_UNSUPPORTED
    assert st(T=5) == E.H3_ERR_EMPTY_PARTITION
    assert st(Cc=7164) == E.H3_ERR_MISALIGNED
    assert st(Cc=0) == E.H3_ERR_INVALID_ARG
    assert st(bias=bias + 2) == E.H3_ERR_MISALIGNED
    assert st(parts=[p + (8 if i == 2 else 0) for i, p in enumerate(parts)]) == E.H3_ERR_MISALIGNED
    assert st(outs=[0] + outs[1:]) == E.H3_ERR_INVALID_ARG
    assert st(outs=[parts[3]] + outs[1:]) == E.H3_ERR_INVALID_ARG      # output over a partial
    assert st(outs=[bias - 64] + outs[1:]) == E.H3_ERR_INVALID_ARG     # output over the bias
    assert st(outs=[outs[0], outs[0] + 256] + outs[2:]) == E.H3_ERR_INVALID_ARG
    assert st(T=2**31) == E.H3_ERR_UNSUPPORTED


def test_binding_rejects_host_tensors():
    x = torch.zeros(4, 3, 8, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        rr.seq_to_head([x], [x.clone()])
    with pytest.raises(ValueError):
        rr.ragged_reduce_scatter([torch.zeros(4, 8, dtype=torch.bfloat16)], None,
                                 [torch.zeros(4, 8, dtype=torch.bfloat16)])


# ---------------------------------------------------------------------------
# staged relayouts: plan and argument checks
# ---------------------------------------------------------------------------

def test_staged_plan_values():
    row = 56 * 128 * 2
    assert rr.staged_plan(32768, 3, 56, 128, 896_000_000) == (32768, 3)
    assert rr.staged_plan(250000, 4, 56, 128, 896_000_000) == (62500, 16)
    assert rr.staged_plan(1000, 3, 56, 128, 7 * row + 100) == (7, 3 * 143)
    assert rr.staged_plan(5, 2, 56, 128, 10 * row) == (5, 2)
    with pytest.raises(rr.H3Error) as e:
        rr.staged_plan(10, 3, 56, 128, row - 16)
    assert e.value.status == _abi.H3_ERR_WINDOW
    with pytest.raises(rr.H3Error) as e:
        rr.staged_plan(0, 3, 56, 128, row)
    assert e.value.status == _abi.H3_ERR_INVALID_ARG


@needs_no_gpu
@pytest.mark.parametrize("fn", ["h3_seq_to_head_staged", "h3_head_to_seq_staged"])
def test_staged_argument_checks(fn):
    T, P, H, D, W = 1000, 3, 56, 128, 6
    send, recv = _layout(T, P, H, D, W)
    if fn == "h3_head_to_seq_staged":
        send, recv = recv, send
    window = BASE - (1 << 30)
    row = H * D * 2
    E = _abi

    def st(window=window, wbytes=64 * row, send=send, recv=recv, W=W, T=T):
        info = _abi.ExecInfo()
        s = getattr(_abi.lib, fn)(_ptrs(send), _ptrs(recv), T, P, H, D, W, C.c_void_p(window),
                                  wbytes, None, C.byref(info))
        assert info.launches == 0
        return s

    assert st(window=0) == E.H3_ERR_INVALID_ARG
    assert st(window=window + 8) == E.H3_ERR_MISALIGNED
    assert st(wbytes=row - 16) == E.H3_ERR_WINDOW
    assert st(wbytes=-1) == E.H3_ERR_INVALID_ARG
    assert st(window=send[2] + 4096) == E.H3_ERR_INVALID_ARG       # window over an input
    assert st(window=recv[0] - 1024, wbytes=4096) == E.H3_ERR_INVALID_ARG  # over an output
    assert st(W=0) == E.H3_ERR_INVALID_ARG
    assert st(T=5) == E.H3_ERR_EMPTY_PARTITION


@needs_no_gpu
def test_all_gather_argument_checks():
    T, Cc, W = 1000, 7168, 6
    addr = BASE
    ins, outs = [], []
    for r in range(W):
        ins.append(addr)
        addr += (T // W + 1) * Cc * 2 + 4096
    for r in range(W):
        outs.append(addr)
        addr += T * Cc * 2 + 4096

    def st(ins=ins, outs=outs, T=T, Cc=Cc, W=W):
        info = _abi.ExecInfo()
        s = _abi.lib.h3_ragged_all_gather(_ptrs(ins), _ptrs(outs), T, Cc, W, None, C.byref(info))
        assert info.launches == 0
        return s

    E = _abi
    assert st(W=0) == E.H3_ERR_INVALID_ARG
    assert st(W=65) == E.H3_ERR_UNSUPPORTED
    assert st(T=5) == E.H3_ERR_EMPTY_PARTITION
    assert st(Cc=7164) == E.H3_ERR_MISALIGNED
    assert st(ins=[ins[0] + 8] + ins[1:]) == E.H3_ERR_MISALIGNED
    assert st(outs=[0] + outs[1:]) == E.H3_ERR_INVALID_ARG
    assert st(outs=[ins[2]] + outs[1:]) == E.H3_ERR_INVALID_ARG
    assert st(outs=[outs[0], outs[0] + 1024] + outs[2:]) == E.H3_ERR_INVALID_ARG


@needs_no_gpu
def test_layout_rejects_unknown_bits():
    T, P, H, D, W = 100, 3, 56, 128, 2
    send, recv = _layout(T, P, H, D, W)
    for layout in (4, 8, -1, 7):
        info = _abi.ExecInfo()
        st = _abi.lib.h3_seq_to_head_layout(_ptrs(send), _ptrs(recv), T, P, H, D, W, 0, layout, None,
                                            None, C.byref(info))
        assert st == _abi.H3_ERR_INVALID_ARG and info.launches == 0
    cfg = _abi.LaunchConfig(_abi.H3_VARIANT_BULK, 0, 0, 0)
    st = _abi.lib.h3_head_to_seq_layout(_ptrs(recv), _ptrs(send), T, P, H, D, W, 0, 2, None,
                                        C.byref(cfg), C.byref(_abi.ExecInfo()))
    assert st == _abi.H3_ERR_UNSUPPORTED


@needs_no_gpu
def test_gated_argument_checks():
    T, Cc, W = 1000, 7168, 6
    addr = BASE
    parts, xs, outs = [], [], []
    for _ in range(W):
        parts.append(addr)
        addr += T * Cc * 2 + 4096
    for r in range(W):
        xs.append(addr)
        addr += (T // W + 1) * Cc * 2 + 4096
    for r in range(W):
        outs.append(addr)
        addr += (T // W + 1) * Cc * 2 + 4096
    gate = addr
    addr += 300 * Cc * 2
    bias = addr

    def st(bounds=(0, 400, 1000), outs=outs, xs=xs, gate=gate, W=W, T=T):
        b = np.asarray(bounds, dtype=np.int64)
        info = _abi.ExecInfo()
        s = _abi.lib.h3_ragged_reduce_scatter_gated(
            _ptrs(parts[:max(W, 0)] + [0] * max(0, W - len(parts))), C.c_void_p(bias), C.c_void_p(gate),
            b.ctypes.data_as(_abi._i64p), len(b) - 1, _ptrs(xs), _ptrs(outs), T, Cc, W, None,
            C.byref(info))
        assert info.launches == 0
        return s

    E = _abi
    assert st(bounds=(0, 400, 400, 1000)) == E.H3_ERR_INVALID_ARG
    assert st(bounds=(1, 400, 1000)) == E.H3_ERR_INVALID_ARG
    assert st(bounds=(0, 400, 999)) == E.H3_ERR_INVALID_ARG
    assert st(bounds=tuple(range(0, 1000, 3)) + (1000,)) == E.H3_ERR_UNSUPPORTED  # 334 segments
    assert st(gate=gate + 8) == E.H3_ERR_MISALIGNED
    assert st(gate=0) == E.H3_ERR_INVALID_ARG
    assert st(outs=[xs[0] + 16] + outs[1:]) == E.H3_ERR_INVALID_ARG   # partial overlap with x
    assert st(outs=[parts[1]] + outs[1:]) == E.H3_ERR_INVALID_ARG
    assert st(outs=[gate] + outs[1:]) == E.H3_ERR_INVALID_ARG
    assert st(outs=[xs[1]] + outs[1:]) == E.H3_ERR_INVALID_ARG          # another rank's x
    assert st(T=5) == E.H3_ERR_EMPTY_PARTITION


@needs_no_gpu
def test_last_cuda_error_is_kept_per_thread():
    """With no GPU a call that reaches the CUDA runtime fails with
    H3_ERR_CUDA; the calling thread's h3_last_cuda_error then holds the CUDA
    error and its text, another thread's stays 0, and the binding's exception
    carries the same error."""
    import threading
    results = {}

    def run():
        msg = C.c_char_p()
        results["fresh"] = _abi.lib.h3_last_cuda_error(C.byref(msg))
        count = C.c_uint32(0)
        results["status"] = _abi.lib.h3_bulk_wait_timeouts(None, C.byref(count), 0)
        results["after"] = _abi.lib.h3_last_cuda_error(C.byref(msg))
        results["text"] = msg.value.decode()
        try:
            _abi.check(results["status"], "h3_bulk_wait_timeouts")
        except _abi.H3Error as e:
            results["exc"] = e

    t = threading.Thread(target=run)
    t.start()
    t.join(timeout=60)
    assert results["fresh"] == 0
    assert results["status"] == _abi.H3_ERR_CUDA
    assert results["after"] != 0 and results["text"] and results["text"] != "no error"
    e = results["exc"]
    assert e.status == _abi.H3_ERR_CUDA and e.cuda_error == results["after"]
    assert results["text"] in str(e)
    other = []
    t2 = threading.Thread(target=lambda: other.append(_abi.lib.h3_last_cuda_error(None)))
    t2.start()
    t2.join(timeout=60)
    assert other == [0]


def _expected_range_plan(T, P, H, D, W, window):
    """Token ranges over all planes, restated from the header's definition:
    one launch if every rank's whole send and receive slices fit; else the
    fewest ranges k and the equal length L = ceil(T_max / k) whose full
    ranges fit (L tokens of P rows sent per rank, W*L tokens of P runs of the
    widest head rank received)."""
    tmax = -(-T // W)
    hmax = -(-H // W)
    send, recv = P * H * D * 2, P * hmax * D * 2
    if tmax * send <= window and T * recv <= window:
        return tmax, 1
    for k in range(2, tmax + 1):
        L = -(-tmax // k)
        if L * send <= window and W * L * recv <= window:
            return L, k
    return None


def test_relayout_range_plan_properties():
    """h3_relayout_chunk_plan_ex with H3_LAUNCH_CHUNK_TOKENS against the
    definition, over a grid of shapes and windows; the windows a one-plane
    plan accepts but that cannot hold one token of every plane are refused;
    without the flag _ex is h3_relayout_chunk_plan; planes per launch."""
    rng = np.random.default_rng(17)
    cases = [(250000, 4, 56, 128, 4), (250000, 4, 56, 128, 2), (32768, 3, 56, 128, 6),
             (131072, 4, 56, 128, 4), (65536, 4, 56, 128, 8), (777, 1, 7, 64, 3)]
    for _ in range(60):
        W = int(rng.integers(1, 9))
        cases.append((int(rng.integers(W, 5000)), int(rng.integers(1, 5)),
                      int(rng.integers(W, 80)), 8 * int(rng.integers(1, 40)), W))
    tok = _abi.H3_LAUNCH_CHUNK_TOKENS
    for T, P, H, D, W in cases:
        tmax, hmax = -(-T // W), -(-H // W)
        row, head = H * D * 2, D * 2
        smallest = P * max(row, W * hmax * head)
        windows = {smallest, smallest + 16, T * P * row, tmax * P * row, tmax * P * row - 16,
                   tmax * row, int(rng.integers(smallest, 4 * tmax * P * row + 1))}
        for win in sorted(windows):
            n, k, per = C.c_int64(0), C.c_int64(0), C.c_int32(0)
            st = _abi.lib.h3_relayout_chunk_plan_ex(T, P, H, D, W, win, tok, C.byref(n), C.byref(k),
                                                    C.byref(per))
            want = _expected_range_plan(T, P, H, D, W, win)
            if win < smallest:
                assert st == _abi.H3_ERR_WINDOW and want is None
                continue
            assert st == _abi.H3_OK and (n.value, k.value) == want, (T, P, H, D, W, win)
            assert per.value == P
            assert rr.relayout_chunk_plan(T, P, H, D, W, win, token_chunks=True) == want
            L, chunks = want
            assert (chunks - 1) * L < tmax <= chunks * L    # exact cover, last range not empty
            if chunks > 1:
                assert L * P * row <= win and W * L * P * hmax * head <= win
        # one token of one plane fits, one token of every plane does not
        if P > 1:
            st = _abi.lib.h3_relayout_chunk_plan_ex(T, P, H, D, W, smallest - 16, tok, C.byref(n),
                                                    C.byref(k), None)
            assert st == _abi.H3_ERR_WINDOW
            assert rr.relayout_chunk_plan(T, P, H, D, W, smallest - 16)[1] >= P
        # flags 0: the one-plane plan; window 0: one launch of all planes either way
        for flags in (0, _abi.H3_LAUNCH_SERIAL):
            win = tmax * row
            st = _abi.lib.h3_relayout_chunk_plan_ex(T, P, H, D, W, win, flags, C.byref(n), C.byref(k),
                                                    C.byref(per))
            assert st == _abi.H3_OK and (n.value, k.value) == rr.relayout_chunk_plan(T, P, H, D, W, win)
            assert per.value == 1
        for flags in (0, tok):
            st = _abi.lib.h3_relayout_chunk_plan_ex(T, P, H, D, W, 0, flags, C.byref(n), C.byref(k),
                                                    C.byref(per))
            assert st == _abi.H3_OK and (n.value, k.value, per.value) == (tmax, 1, P)


def test_relayout_range_plan_rejects_bad_arguments():
    n, k = C.c_int64(0), C.c_int64(0)
    f = _abi.lib.h3_relayout_chunk_plan_ex
    for flags in (4, -1, _abi.H3_LAUNCH_CHUNK_TOKENS | 8):
        assert f(1000, 3, 56, 128, 4, 10 ** 9, flags, C.byref(n), C.byref(k), None) == _abi.H3_ERR_INVALID_ARG
    assert f(1000, 3, 56, 128, 4, 10 ** 9, 2, None, C.byref(k), None) == _abi.H3_ERR_INVALID_ARG
    assert f(1000, 3, 56, 128, 4, 10 ** 9, 2, C.byref(n), None, None) == _abi.H3_ERR_INVALID_ARG
    assert f(1000, 0, 56, 128, 4, 10 ** 9, 2, C.byref(n), C.byref(k), None) == _abi.H3_ERR_INVALID_ARG
    assert f(1000, 3, 56, 128, 4, -1, 2, C.byref(n), C.byref(k), None) == _abi.H3_ERR_INVALID_ARG
    assert f(3, 3, 56, 128, 4, 10 ** 9, 2, C.byref(n), C.byref(k), None) == _abi.H3_ERR_EMPTY_PARTITION


@needs_no_gpu
def test_relayout_range_window_check_long_workload():
    """250k QKVG over 4 ranks: the pages' window holds one plane of one rank
    and equally 15,625 tokens of all four planes, so both shapes take 4
    launches; a window below one token of every plane is refused by the
    range shape before anything is launched, though one plane per launch
    still fits it."""
    T, P, H, D, W = 250000, 4, 56, 128, 4
    send, recv = _layout(T, P, H, D, W)
    assert 15625 * 4 * 56 * 128 * 2 == 896_000_000
    assert rr.relayout_chunk_plan(T, P, H, D, W, 896_000_000, token_chunks=True) == (15625, 4)
    assert rr.relayout_chunk_plan(T, P, H, D, W, 896_000_000 - 16, token_chunks=True) == (12500, 5)
    small = P * H * D * 2 - 16
    cfg = C.byref(_abi.LaunchConfig(0, 0, _abi.H3_LAUNCH_CHUNK_TOKENS, 0))
    for fn in ("h3_seq_to_head_ex", "h3_head_to_seq_ex"):
        info = _abi.ExecInfo()
        st = getattr(_abi.lib, fn)(_ptrs(send), _ptrs(recv), T, P, H, D, W, small, None, cfg,
                                   C.byref(info))
        assert st == _abi.H3_ERR_WINDOW and info.launches == 0, fn
    assert rr.relayout_chunk_plan(T, P, H, D, W, small)[1] > P


def test_token_chunks_cover_every_token_once():
    """The token chunks a chunked relayout launches, as the header defines
    them: chunk c of a plane holds local tokens [c*L, c*L + L) of every rank
    (fewer in the last chunk, possibly none for a smaller rank).  Over many
    random shapes and windows, mapping each launch's token units to (rank,
    local token) by the chunk's quotient/remainder split covers every token
    of every rank exactly once, and every launch's per-rank slices fit the
    window."""
    rng = np.random.default_rng(11)
    checked_empty_rank = False
    for _ in range(400):
        W = int(rng.integers(1, 17))
        T = int(rng.integers(W, 3000))
        H = int(rng.integers(W, 90))
        D = 8 * int(rng.integers(1, 33))
        P = int(rng.integers(1, 5))
        row, head = H * D * 2, D * 2
        part = rr.partition(T, H, W)
        tq, tm = divmod(T, W)
        hmax = max(part.heads(j) for j in range(W))
        smallest = max(row, W * hmax * head)
        window = int(rng.integers(smallest, (tq + 1) * row * 2 + 1))
        L, chunks = rr.relayout_chunk_plan(T, P, H, D, W, window)
        k = chunks // P
        assert chunks == k * P and k >= 1
        seen = {}
        for c in range(k):
            t0 = c * L
            cq, cm = (L, 0) if c + 1 < k else (tq - t0, tm)
            assert cq >= 0 and cq * W + cm > 0           # no empty launch
            if cq == 0:
                checked_empty_rank = True
            counts = [0] * W
            for v in range(cq * W + cm):
                big = cm * (cq + 1)                      # owner under the chunk's split
                s = v // (cq + 1) if v < big else cm + (v - big) // cq
                start = s * cq + min(s, cm)
                tl = t0 + v - start
                assert 0 <= tl < part.tokens(s)
                assert (s, tl) not in seen
                seen[(s, tl)] = c
                counts[s] += 1
            # this launch's slices: each rank sends its tokens, each head rank
            # receives every rank's tokens of its heads
            assert max(counts) * row <= window
            assert sum(counts) * hmax * head <= window
        assert len(seen) == T
    assert checked_empty_rank  # some last chunk left a smaller rank without tokens


@needs_no_gpu
def test_relayout_sides_beyond_the_byte_limit_are_refused():
    """A relayout side of T*P*H*D*2 bytes above 2^56 (rows and row width each
    within their own limits) is refused with H3_ERR_UNSUPPORTED by every
    relayout entry point and the plan queries, before any byte count could
    leave 64 bits; just below the limit the plan query answers."""
    W = 2
    send = [BASE + r * (1 << 50) for r in range(W)]   # made-up, never dereferenced
    recv = [BASE + (4 + r) * (1 << 50) for r in range(W)]
    n, k = C.c_int64(0), C.c_int64(0)
    plan = _abi.lib.h3_relayout_chunk_plan_ex
    for T, P, H, D in ((1 << 30, 1, 1 << 16, 1 << 14), (1 << 28, 4, 1 << 16, 1 << 14),
                       ((1 << 31) - 1, 1, 1 << 15, 1 << 14)):
        assert T * P * H * D * 2 > 1 << 56 and T * P < 2 ** 31 and H * D * 2 // 16 <= 1 << 30
        for flags in (0, _abi.H3_LAUNCH_CHUNK_TOKENS):
            assert plan(T, P, H, D, W, 10 ** 9, flags, C.byref(n), C.byref(k), None) == _abi.H3_ERR_UNSUPPORTED
        assert _abi.lib.h3_relayout_chunk_plan(T, P, H, D, W, 0, C.byref(n), C.byref(k)) == _abi.H3_ERR_UNSUPPORTED
        for fn in ("h3_seq_to_head", "h3_head_to_seq"):
            st, info = _relayout_status(send, recv, T, P, H, D, W, fn=fn)
            assert st == _abi.H3_ERR_UNSUPPORTED and info.launches == 0, (fn, T, P)
        for fn in ("h3_seq_to_head_rank", "h3_head_to_seq_rank"):
            info = _abi.ExecInfo()
            st = getattr(_abi.lib, fn)(_ptrs(send), C.c_void_p(recv[0]), T, P, H, D, W, 0, 0, None,
                                       None, C.byref(info))
            assert st == _abi.H3_ERR_UNSUPPORTED and info.launches == 0, (fn, T, P)
    # 2^55 bytes a side: within the limit
    assert plan(1 << 30, 1, 1 << 10, 1 << 14, W, 10 ** 9, 0, C.byref(n), C.byref(k), None) == _abi.H3_OK
    # a head row that is not whole 16-byte vectors, through the plan query too
    assert plan(1000, 3, 56, 4, W, 10 ** 9, 0, C.byref(n), C.byref(k), None) == _abi.H3_ERR_MISALIGNED


@needs_no_gpu
def test_row_calls_beyond_the_byte_limit_are_refused():
    """Reduce-scatter, gated reduce-scatter, all-gather and their rank calls
    refuse T*C*2 above 2^56 bytes (T and C/8 each within their own limits)
    with H3_ERR_UNSUPPORTED before anything is launched."""
    W, T, Cc = 2, (1 << 31) - 1, 1 << 28
    assert T * Cc * 2 > 1 << 56 and Cc // 8 <= 1 << 30
    full = [BASE + r * (1 << 52) for r in range(W)]   # made-up, never dereferenced
    blocks = [BASE + (4 + r) * (1 << 52) for r in range(W)]
    info = _abi.ExecInfo()
    assert _abi.lib.h3_ragged_reduce_scatter(_ptrs(full), None, _ptrs(blocks), T, Cc, W, None,
                                             C.byref(info)) == _abi.H3_ERR_UNSUPPORTED
    assert _abi.lib.h3_ragged_all_gather(_ptrs(blocks), _ptrs(full), T, Cc, W, None,
                                         C.byref(info)) == _abi.H3_ERR_UNSUPPORTED
    assert _abi.lib.h3_ragged_reduce_scatter_rank(_ptrs(full), None, C.c_void_p(blocks[0]), T, Cc, W, 0,
                                                  None, None, C.byref(info)) == _abi.H3_ERR_UNSUPPORTED
    assert _abi.lib.h3_ragged_all_gather_rank(_ptrs(blocks), C.c_void_p(full[0]), T, Cc, W, 0, None,
                                              None, C.byref(info)) == _abi.H3_ERR_UNSUPPORTED
    assert info.launches == 0


def test_relayout_launch_plan_dict():
    """The binding's full plan query: tokens per launch, launches and planes
    per launch for the three cuts of the 250k QKVG operand over 4 ranks."""
    T, P, H, D, W = 250000, 4, 56, 128, 4
    assert rr.relayout_launch_plan(T, P, H, D, W, 0) == \
        {"tokens_per_launch": 62500, "launches": 1, "planes_per_launch": 4}
    assert rr.relayout_launch_plan(T, P, H, D, W, 896_000_000) == \
        {"tokens_per_launch": 62500, "launches": 4, "planes_per_launch": 1}
    assert rr.relayout_launch_plan(T, P, H, D, W, 896_000_000, token_chunks=True) == \
        {"tokens_per_launch": 15625, "launches": 4, "planes_per_launch": 4}
    with pytest.raises(rr.H3Error):
        rr.relayout_launch_plan(T, P, H, D, W, P * H * D * 2 - 16, token_chunks=True)
