"""The staged seq->head relayout that allocates no device memory.

Some callers cannot allocate device memory themselves -- for example a plugin
that only receives tensors from a host framework whose caching allocator owns
the whole memory budget, or a latency-critical loop in which cudaMalloc or
cudaFree would synchronise the device.  For them the library offers
h3_seq_to_head_staged_noalloc: the staged seq->head relayout with its staging
window in a fixed 16 MiB device array inside the library.

This test calls that entry point through the C ABI twice in a row, on
different inputs and window sizes, and compares each result with the existing
entry point h3_seq_to_head_staged (given a window this test allocates) bit
for bit, the tolerance every relayout test uses.  The second call also shows
that what the first call left in the shared array does not leak into the next
result.  Another test checks the property the entry point exists for: once
its first call has set it up (that call loads the array), repeated calls leave
the device's free memory, as cudaMemGetInfo reports it, unchanged.  The file
is collected after every other test and passes both alone in a fresh process
and after the rest of the suite.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import ragged_reduce_b200 as rr
import workloads as wl
from ragged_reduce_b200 import _abi
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

DEV = "cuda"
STATIC_WINDOW_BYTES = 16 << 20


def _noalloc():
    f = _abi.lib.h3_seq_to_head_staged_noalloc
    f.restype = C.c_int
    f.argtypes = [C.POINTER(C.c_void_p), C.POINTER(C.c_void_p), C.c_int64, C.c_int32, C.c_int32,
                  C.c_int32, C.c_int32, C.c_int64, C.c_void_p, C.POINTER(_abi.ExecInfo)]
    return f


def _case(T, P, H, D, W, seed):
    full = wl.random_bits((T, P, H, D), seed, DEV)
    part = rr.partition(T, H, W)
    return full, rr.split_rows(full, part.token_starts)


def _call_noalloc(send, recv, T, P, H, D, W, window_bytes):
    info = _abi.ExecInfo()
    stream = torch.cuda.current_stream().cuda_stream
    st = _noalloc()(_abi.pointer_array([s.data_ptr() for s in send]),
                    _abi.pointer_array([r.data_ptr() for r in recv]),
                    T, P, H, D, W, window_bytes, C.c_void_p(stream), C.byref(info))
    return st, info


@pytest.mark.parametrize("first,second", [
    # (T, P, H, D, W, window bytes, seed): many small chunks, then the whole array
    ((1000, 3, 56, 128, 6, 7 * 14336 + 100, 11), (777, 4, 56, 128, 8, 0, 12)),
    ((2500, 2, 56, 128, 4, 0, 13), (130, 2, 7, 64, 3, 5 * 896, 14)),
])
def test_noalloc_matches_staged_twice(first, second):
    for T, P, H, D, W, window_bytes, seed in (first, second):
        full, send = _case(T, P, H, D, W, seed)
        got = rr.alloc_head_side(T, P, H, D, W, DEV)
        for g in got:
            g.view(torch.int16).fill_(0x5A5A)  # stale pattern that must be overwritten
        st, info = _call_noalloc(send, got, T, P, H, D, W, window_bytes)
        assert st == _abi.H3_OK, _abi.describe(st)
        used = window_bytes or STATIC_WINDOW_BYTES
        n_tok, chunks = rr.staged_plan(T, P, H, D, used)
        assert info.chunks == chunks and info.launches == 2 * chunks
        # the existing entry point, on a window of the same size
        want = rr.alloc_head_side(T, P, H, D, W, DEV)
        window = torch.empty(used, dtype=torch.uint8, device=DEV)
        rr.seq_to_head_staged(send, want, window)
        torch.cuda.synchronize()
        for j in range(W):
            assert np.array_equal(gu.bits(got[j]), gu.bits(want[j])), f"rank {j}"
        # and both equal the direct relayout
        direct = rr.alloc_head_side(T, P, H, D, W, DEV)
        rr.seq_to_head(send, direct)
        for j in range(W):
            assert gu.same_bits(got[j], direct[j])


def test_noalloc_rejects_window_beyond_its_array():
    T, P, H, D, W = 64, 3, 56, 128, 2
    full, send = _case(T, P, H, D, W, 15)
    recv = rr.alloc_head_side(T, P, H, D, W, DEV)
    st, info = _call_noalloc(send, recv, T, P, H, D, W, STATIC_WINDOW_BYTES + 16)
    assert st == _abi.H3_ERR_UNSUPPORTED and info.launches == 0
    st, info = _call_noalloc(send, recv, T, P, H, D, W, 14336 - 16)
    assert st == _abi.H3_ERR_WINDOW and info.launches == 0


def test_noalloc_calls_leave_device_memory_unchanged():
    """The point of the entry point: once set up, calls change no device
    memory use.  Every buffer is allocated first and one round of calls loads
    the array and the kernels; after that, two more rounds of both shapes must
    leave cudaMemGetInfo's free bytes exactly as they were, and still match
    the staged call."""
    shapes = [(1000, 3, 56, 128, 6, 7 * 14336 + 100, 21), (777, 4, 56, 128, 8, 0, 22)]
    cases = []
    for T, P, H, D, W, window_bytes, seed in shapes:
        full, send = _case(T, P, H, D, W, seed)
        got = rr.alloc_head_side(T, P, H, D, W, DEV)
        want = rr.alloc_head_side(T, P, H, D, W, DEV)
        window = torch.empty(window_bytes or STATIC_WINDOW_BYTES, dtype=torch.uint8, device=DEV)
        rr.seq_to_head_staged(send, want, window)
        cases.append((T, P, H, D, W, window_bytes, full, send, got, want))

    def one_round():
        for T, P, H, D, W, window_bytes, _, send, got, _ in cases:
            st, _ = _call_noalloc(send, got, T, P, H, D, W, window_bytes)
            assert st == _abi.H3_OK, _abi.describe(st)

    def stale_outputs():
        for case in cases:
            for g in case[8]:
                g.view(torch.int16).fill_(0x5A5A)  # must be overwritten

    one_round()  # set-up: the array and the kernels are loaded here
    stale_outputs()  # and the fill kernel, before the measurement
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for _ in range(2):
        stale_outputs()
        one_round()
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before, (free_before, free_after)
    for T, P, H, D, W, _, _, _, got, want in cases:
        for j in range(W):
            assert gu.same_bits(got[j], want[j]), f"rank {j}"
