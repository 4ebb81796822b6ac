"""Programmatic dependent launch keeps stream order.

By default the relayout kernels may be scheduled while the previous kernel in
the stream drains; each waits for it before touching memory, and the later
plane launches of a chunked call wait for the previous plane at their end.
These tests chain dependent calls on one stream (every call reads what the
previous one wrote) and check every result bit for bit, with programmatic
launch on and off (H3_LAUNCH_SERIAL)."""
import numpy as np
import pytest
import torch

import ragged_reduce_b200 as rr
import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.mark.parametrize("chunked", [None, "plane", "sub"])
def test_serial_and_programmatic_launches_agree(oracle_lib, chunked):
    T, P, H, D, W = 1000, 4, 56, 128, 6
    part = rr.partition(T, H, W)
    x = wl.random_bits((T, P, H, D), 71, DEV)
    send = rr.split_rows(x, part.token_starts)
    window = gu.chunk_window(chunked, T, H, D, W)
    outs = {}
    for serial in (False, True):
        heads = rr.alloc_head_side(T, P, H, D, W, DEV)
        info = rr.seq_to_head(send, heads, window_bytes=window, serial=serial)
        assert info["launches"] == rr.relayout_chunk_plan(T, P, H, D, W, window)[1]
        back_full, back = rr.alloc_seq_side(T, P, H, D, W, DEV)
        rr.head_to_seq(heads, back, window_bytes=window, serial=serial)
        outs[serial] = (heads, back_full)
    want = oracle_lib.seq_to_head([gu.bits(s) for s in send], T, P, H, D, W)
    for serial, (heads, back_full) in outs.items():
        for j in range(W):
            assert np.array_equal(gu.bits(heads[j]), want[j]), (serial, j)
        assert gu.same_bits(back_full, x), serial


@pytest.mark.parametrize("serial", [False, True])
@pytest.mark.parametrize("chunked", ["plane", "sub", "ranges"])
def test_chained_dependent_calls(oracle_lib, serial, chunked):
    """x -> heads -> back -> heads2 -> back2, all chunked (one plane per
    launch, every plane in token chunks, or token ranges of all planes), on
    one stream, with a fresh x written by a PyTorch kernel before every
    round."""
    T, P, H, D, W = 4096, 4, 56, 128, 6
    part = rr.partition(T, H, W)
    x = torch.empty((T, P, H, D), dtype=torch.bfloat16, device=DEV)
    send = rr.split_rows(x, part.token_starts)
    heads = rr.alloc_head_side(T, P, H, D, W, DEV)
    heads2 = rr.alloc_head_side(T, P, H, D, W, DEV)
    back_full, back = rr.alloc_seq_side(T, P, H, D, W, DEV)
    back2_full, back2 = rr.alloc_seq_side(T, P, H, D, W, DEV)
    ranges = chunked == "ranges"
    if ranges:
        window = gu.range_window("plane", T, P, H, D, W) // 3  # about twelve ranges
        assert rr.relayout_chunk_plan(T, P, H, D, W, window, token_chunks=True)[1] >= 10
    else:
        window = gu.chunk_window(chunked, T, H, D, W)
    if chunked == "sub":
        window //= 3  # about six token chunks per plane: long chains of launches
        assert rr.relayout_chunk_plan(T, P, H, D, W, window)[1] >= 5 * P
    kw = dict(window_bytes=window, serial=serial, token_chunks=ranges)
    for round_ in range(8):
        x.copy_(wl.random_bits((T, P, H, D), 500 + round_, DEV))
        rr.seq_to_head(send, heads, **kw)
        rr.head_to_seq(heads, back, **kw)
        rr.seq_to_head(back, heads2, **kw)
        rr.head_to_seq(heads2, back2, **kw)
        assert gu.same_bits(back_full, x), round_
        assert gu.same_bits(back2_full, x), round_
        for j in range(W):
            assert gu.same_bits(heads2[j], heads[j]), (round_, j)
        if round_ == 0:
            want = oracle_lib.seq_to_head([gu.bits(s) for s in send], T, P, H, D, W)
            for j in range(W):
                assert np.array_equal(gu.bits(heads[j]), want[j]), j


def test_prepared_serial_option():
    T, P, H, D, W = 700, 3, 56, 128, 4
    part = rr.partition(T, H, W)
    x = wl.random_bits((T, P, H, D), 73, DEV)
    send = rr.split_rows(x, part.token_starts)
    heads = rr.alloc_head_side(T, P, H, D, W, DEV)
    back_full, back = rr.alloc_seq_side(T, P, H, D, W, DEV)
    window = max(part.tokens(0) * H * D * 2, T * part.heads(0) * D * 2)
    fwd = rr.prepare_seq_to_head(send, heads, window_bytes=window, serial=True)
    bwd = fwd.inverse(heads, back)
    assert bwd.serial
    fwd()
    bwd()
    assert gu.same_bits(back_full, x)


@pytest.mark.parametrize("serial", [False, True])
def test_chained_reduce_gather_gated(oracle_lib, serial):
    """reduce-scatter -> all-gather of its rows -> gated reduce-scatter in
    place on a residual that a relayout round trip just rewrote, on one
    stream, every round with fresh partials."""
    T, C, W, S = 3000, 2048, 6, 5
    part = rr.partition(T, W, W)
    partials = torch.empty((W, T, C), dtype=torch.bfloat16, device=DEV)
    bias = wl.normal_bf16((C,), 81, 0.1, DEV)
    red_full, red = rr.alloc_reduce_outputs(T, C, W, DEV)
    gath = [torch.empty((T, C), dtype=torch.bfloat16, device=DEV) for _ in range(W)]
    gate = wl.normal_bf16((S, C), 82, 1.0, DEV)
    bounds = wl.segment_bounds(T, S, 83)
    x_src = wl.normal_bf16((T, C), 84, 1.0, DEV)
    x_full = torch.empty_like(x_src)
    x = rr.split_rows(x_full, part.token_starts)
    for round_ in range(4):
        partials.copy_(wl.normal_bf16((W, T, C), 90 + round_, 0.5, DEV))
        x_full.copy_(x_src)
        rr.ragged_reduce_scatter(partials, bias, red, serial=serial)
        rr.ragged_all_gather(red, gath, serial=serial)
        rr.ragged_reduce_scatter_gated(partials, bias, gate, bounds, x)
        want = oracle_lib.ragged_reduce_scatter([gu.bits(p) for p in partials.unbind(0)],
                                                gu.bits(bias), W)
        for r in range(W):
            assert np.array_equal(gu.bits(red[r]), want[r]), (round_, r)
        for g in gath:
            assert gu.same_bits(g, red_full), round_
        want_g = oracle_lib.reduce_scatter_gated(
            [gu.bits(p) for p in partials.unbind(0)], gu.bits(bias), gu.bits(gate), bounds,
            [gu.bits(v) for v in rr.split_rows(x_src, part.token_starts)], W)
        for r in range(W):
            assert np.array_equal(gu.bits(x[r]), want_g[r]), (round_, r)


def test_staged_calls_chain_on_one_stream(oracle_lib):
    """Staged calls through a 37-row window (330 launches per call, each
    reading what the previous one wrote or overwriting the window it read),
    chained with direct relayouts and torch copies on one stream, fresh data
    every round: the programmatic launches must keep stream order."""
    T, P, H, D, W = 2000, 3, 56, 128, 6
    part = rr.partition(T, H, W)
    full = torch.empty((T, P, H, D), dtype=torch.bfloat16, device=DEV)
    send = rr.split_rows(full, part.token_starts)
    heads = rr.alloc_head_side(T, P, H, D, W, DEV)
    heads2 = rr.alloc_head_side(T, P, H, D, W, DEV)
    back_full, back = rr.alloc_seq_side(T, P, H, D, W, DEV)
    win = torch.empty(37 * H * D * 2, dtype=torch.uint8, device=DEV)
    assert rr.staged_plan(T, P, H, D, win.numel())[1] == 3 * 55
    for round_ in range(4):
        src = wl.random_bits((T, P, H, D), 300 + round_, DEV)
        full.copy_(src)
        info = rr.seq_to_head_staged(send, heads, win)
        assert info["launches"] == 330
        rr.head_to_seq(heads, back)
        rr.seq_to_head_staged(back, heads2, win)
        rr.head_to_seq_staged(heads2, back, win)
        want = oracle_lib.seq_to_head([gu.bits(s) for s in send], T, P, H, D, W)
        for j in range(W):
            assert np.array_equal(gu.bits(heads2[j]), want[j]), (round_, j)
        assert gu.same_bits(back_full, src), round_
