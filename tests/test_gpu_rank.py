"""One rank per GPU, checked on one GPU: the W rank calls together must write
exactly what the one-GPU call writes ("Distributed H3 Execution", "Remaining
GPU Gates": distributed-versus-single parity).  Every rank's buffers sit in
this GPU's memory and are passed as plain device addresses, the form peers'
mapped buffers take; each call writes only its rank's output."""
import numpy as np
import pytest
import torch

import ragged_reduce_b200 as rr
import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

DEV = "cuda"

SHAPES = [  # T, P, H, D, W
    (1024, 3, 56, 128, 2), (1000, 3, 56, 128, 6), (777, 4, 56, 128, 4), (513, 1, 56, 128, 8),
    (300, 2, 30, 64, 7), (97, 3, 9, 8, 3), (200, 2, 56, 128, 1), (129, 1, 64, 256, 5),
    # head runs longer than a CTA's slots (32 KB and 20 KB): the long-run pull kernel
    (50, 2, 64, 256, 1), (60, 2, 40, 512, 2),
]


@pytest.mark.parametrize("T,P,H,D,W", SHAPES)
@pytest.mark.parametrize("chunked", [None, "plane", "sub", "ranges"])
def test_relayout_rank_shares(oracle_lib, T, P, H, D, W, chunked):
    part = rr.partition(T, H, W)
    x = wl.random_bits((T, P, H, D), T + W, DEV)
    send = rr.split_rows(x, part.token_starts)
    addrs = [int(s.data_ptr()) for s in send]
    ranges = chunked == "ranges"  # token ranges of every plane (H3_LAUNCH_CHUNK_TOKENS)
    window = gu.range_window("half", T, P, H, D, W) if ranges else gu.chunk_window(chunked, T, H, D, W)
    L, chunks = rr.relayout_chunk_plan(T, P, H, D, W, window, token_chunks=ranges)
    heads = [torch.empty((T, P, part.heads(k), D), dtype=torch.bfloat16, device=DEV)
             for k in range(W)]
    for k in range(W):
        info = rr.seq_to_head_rank(addrs, heads[k], k, n_heads=H, window_bytes=window,
                                   token_chunks=ranges)
        assert info["chunks"] == chunks and info["launches"] == chunks
    want = oracle_lib.seq_to_head([gu.bits(s) for s in send], T, P, H, D, W)
    for k in range(W):
        assert np.array_equal(gu.bits(heads[k]), want[k]), (T, P, H, D, W, k)
    back_full, back = rr.alloc_seq_side(T, P, H, D, W, DEV)
    head_addrs = [int(h.data_ptr()) for h in heads]
    for k in range(W):
        info = rr.head_to_seq_rank(head_addrs, back[k], k, n_tokens=T, window_bytes=window,
                                   token_chunks=ranges)
        # launches: the chunks that hold tokens of rank k
        groups = P if window and not ranges else 1
        per_group = chunks // groups
        held = sum(1 for c in range(per_group) if c * L < part.tokens(k))
        assert info["chunks"] == chunks and info["launches"] == held * groups
    assert gu.same_bits(back_full, x)


def test_relayout_rank_matches_full_call_at_bench_size():
    T, P, H, D, W = 32768, 3, 56, 128, 6
    part = rr.partition(T, H, W)
    x = wl.normal_bf16((T, P, H, D), 2, 1.0, DEV)
    send = rr.split_rows(x, part.token_starts)
    full = rr.alloc_head_side(T, P, H, D, W, DEV)
    rr.seq_to_head(send, full)
    for k in range(W):
        mine = torch.empty_like(full[k])
        rr.seq_to_head_rank(send, mine, k, n_heads=H, window_bytes=896_000_000)
        assert gu.same_bits(mine, full[k]), k
    back_full, back = rr.alloc_seq_side(T, P, H, D, W, DEV)
    for k in range(W):
        rr.head_to_seq_rank(full, back[k], k, n_tokens=T)
    assert gu.same_bits(back_full, x)


@pytest.mark.parametrize("T,C,W", [(1000, 7168, 6), (1024, 7168, 8), (97, 2048, 2), (129, 8, 5),
                                   (70, 256, 16), (64, 64, 64), (50, 4104, 1)])
@pytest.mark.parametrize("with_bias", [True, False])
def test_reduce_and_gather_rank_shares(oracle_lib, T, C, W, with_bias):
    w = wl.ReduceWorkload("r", T=T, C=C, W=W, seed=T * 3 + W)
    partials, bias = wl.partials_and_bias(w, DEV)
    bias = bias if with_bias else None
    part = rr.partition(T, W, W)
    outs = [torch.empty((part.tokens(k), C), dtype=torch.bfloat16, device=DEV) for k in range(W)]
    addrs = [int(p.data_ptr()) for p in partials.unbind(0)]
    for k in range(W):
        rr.ragged_reduce_scatter_rank(addrs, bias, outs[k], k, n_tokens=T)
    want = oracle_lib.ragged_reduce_scatter([gu.bits(p) for p in partials.unbind(0)],
                                            None if bias is None else gu.bits(bias), W)
    for k in range(W):
        assert np.array_equal(gu.bits(outs[k]), want[k]), (T, C, W, k)
    gathered = [torch.empty((T, C), dtype=torch.bfloat16, device=DEV) for _ in range(W)]
    for k in range(W):
        rr.ragged_all_gather_rank(outs, gathered[k], k)
    expect = torch.cat(outs, 0)
    for g in gathered:
        assert gu.same_bits(g, expect)


def test_reduce_rank_random_bit_patterns(oracle_lib):
    T, C, W = 300, 1024, 5
    partials = wl.random_bits((W, T, C), 41, DEV)
    bias = wl.random_bits((C,), 42, DEV)
    part = rr.partition(T, W, W)
    want = oracle_lib.ragged_reduce_scatter([gu.bits(p) for p in partials], gu.bits(bias), W)
    for k in range(W):
        out = torch.empty((part.tokens(k), C), dtype=torch.bfloat16, device=DEV)
        rr.ragged_reduce_scatter_rank(list(partials.unbind(0)), bias, out, k, n_tokens=T)
        assert gu.nan_aware_equal(gu.bits(out), want[k]).all(), k


def test_rank_calls_serial_and_guard_bands(oracle_lib):
    """Serial launches give the same bytes; nothing outside a rank's output
    is written."""
    T, P, H, D, W = 600, 3, 56, 128, 4
    part = rr.partition(T, H, W)
    x = wl.random_bits((T, P, H, D), 43, DEV)
    send = rr.split_rows(x, part.token_starts)
    want = oracle_lib.seq_to_head([gu.bits(s) for s in send], T, P, H, D, W)
    for k in range(W):
        buf, mine = gu.guarded((T, P, part.heads(k), D), DEV)
        rr.seq_to_head_rank(send, mine, k, n_heads=H, serial=True)
        assert gu.guards_intact(buf)
        assert np.array_equal(gu.bits(mine), want[k])
    heads = [torch.from_numpy(want[k].view(np.int16)).view(torch.bfloat16).to(DEV) for k in range(W)]
    for k in range(W):
        buf, mine = gu.guarded((part.tokens(k), P, H, D), DEV)
        rr.head_to_seq_rank(heads, mine, k, n_tokens=T)
        assert gu.guards_intact(buf)
        assert gu.same_bits(mine, send[k])


@pytest.mark.parametrize("T,C,W,S", [(1000, 7168, 6, 8), (1024, 2048, 8, 3), (97, 1024, 2, 1),
                                     (300, 256, 5, 40), (64, 64, 64, 64), (777, 512, 4, 256)])
def test_gated_rank_shares(oracle_lib, T, C, W, S):
    """Each rank's gated rows, in place on its residual, from the clipped and
    rebased segments of its own token range."""
    w = wl.ReduceWorkload("g", T=T, C=C, W=W, seed=T + S)
    partials, bias = wl.partials_and_bias(w, DEV)
    gate = wl.normal_bf16((S, C), S, 1.0, DEV)
    bounds = wl.segment_bounds(T, S, S + 1)
    part = rr.partition(T, W, W)
    x_full = wl.normal_bf16((T, C), S + 2, 1.0, DEV)
    x_bits = [gu.bits(v) for v in rr.split_rows(x_full, part.token_starts)]
    xs = [v.clone() for v in rr.split_rows(x_full, part.token_starts)]
    for k in range(W):
        rr.ragged_reduce_scatter_gated_rank(list(partials.unbind(0)), bias, gate, bounds, xs[k], k,
                                            n_tokens=T)
    want = oracle_lib.reduce_scatter_gated([gu.bits(p) for p in partials.unbind(0)], gu.bits(bias),
                                           gu.bits(gate), bounds, x_bits, W)
    for k in range(W):
        assert np.array_equal(gu.bits(xs[k]), want[k]), (T, C, W, S, k)
    # out of place into a guarded buffer gives the same rows and writes nothing else
    k = W - 1
    buf, out = gu.guarded((part.tokens(k), C), DEV)
    x_k = rr.split_rows(x_full, part.token_starts)[k]
    rr.ragged_reduce_scatter_gated_rank(list(partials.unbind(0)), bias, gate, bounds, x_k, k,
                                        n_tokens=T, out=out)
    assert gu.guards_intact(buf)
    assert np.array_equal(gu.bits(out), want[k])


def test_rank_reduce_calls_refuse_non_bf16_tensors():
    """float16 (or int16) tensors would be read as BF16 bits: the rank reduce
    wrappers refuse them before anything is launched, as the one-GPU calls do."""
    T, C, W = 64, 64, 2
    partials = [torch.zeros((T, C), dtype=torch.bfloat16, device=DEV) for _ in range(W)]
    out = torch.empty((32, C), dtype=torch.bfloat16, device=DEV)
    gate = torch.zeros((1, C), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ValueError, match="BF16"):
        rr.ragged_reduce_scatter_rank(partials, None, out.half(), 0, n_tokens=T)
    with pytest.raises(ValueError, match="BF16"):
        rr.ragged_reduce_scatter_rank([p.half() for p in partials], None, out, 0, n_tokens=T)
    with pytest.raises(ValueError, match="BF16"):
        rr.ragged_reduce_scatter_gated_rank(partials, None, gate, [0, T], out.half(), 0, n_tokens=T)
    with pytest.raises(ValueError, match="BF16"):
        rr.ragged_reduce_scatter_gated_rank(partials, None, gate.half(), [0, T], out, 0, n_tokens=T)
