"""Buffers 16- but not 32-byte aligned: every call must take its 16-byte
kernels (the 32-byte ones need every pointer 32-byte aligned) and still equal
the oracle bit for bit.  One buffer per call sits at an address that is 16
modulo 32 (a view 16 bytes into a larger allocation)."""
import numpy as np
import pytest
import torch

import ragged_reduce_b200 as rr
import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _off16(src: torch.Tensor) -> torch.Tensor:
    """A copy of `src` at an address that is 16 modulo 32."""
    nbytes = src.numel() * src.element_size()
    buf = torch.empty(nbytes + 64, dtype=torch.uint8, device=DEV)
    base = buf.data_ptr() % 32
    start = (16 - base) % 32
    view = buf[start:start + nbytes].view(src.dtype).view(src.shape)
    view.copy_(src)
    assert view.data_ptr() % 32 == 16
    return view


@pytest.mark.parametrize("window", [0, "plane", "ranges"])
@pytest.mark.parametrize("which", ["send", "recv"])
def test_relayouts_with_a_16_byte_aligned_buffer(oracle_lib, window, which):
    T, P, H, D, W = 300, 3, 56, 128, 4
    part = rr.partition(T, H, W)
    full = wl.random_bits((T, P, H, D), 7 + len(which), DEV)
    send = [t.clone() for t in rr.split_rows(full, part.token_starts)]
    heads = rr.alloc_head_side(T, P, H, D, W, DEV)
    if which == "send":
        send[1] = _off16(send[1])
    else:
        heads[2] = _off16(heads[2])
    tok = window == "ranges"
    wb = {0: 0, "plane": gu.chunk_window("plane", T, H, D, W),
          "ranges": gu.range_window("half", T, P, H, D, W)}[window]
    rr.seq_to_head(send, heads, window_bytes=wb, token_chunks=tok)
    want = oracle_lib.seq_to_head([gu.bits(s) for s in send], T, P, H, D, W)
    for j in range(W):
        assert np.array_equal(gu.bits(heads[j]), want[j]), j
    back = [torch.empty_like(s) for s in send]
    if which == "recv":
        back[3] = _off16(back[3])
    rr.head_to_seq(heads, back, window_bytes=wb, token_chunks=tok)
    for r in range(W):
        assert gu.same_bits(back[r], send[r]), r


def test_row_calls_with_16_byte_aligned_buffers(oracle_lib):
    T, C, W, S = 333, 7168, 6, 5
    w = wl.ReduceWorkload("a", T=T, C=C, W=W, seed=77)
    partials, bias = wl.partials_and_bias(w, DEV)
    plist = [p.clone() for p in partials.unbind(0)]
    plist[4] = _off16(plist[4])
    bias16 = _off16(bias)
    part = rr.partition(T, W, W)
    out = [torch.empty((part.tokens(r), C), dtype=torch.bfloat16, device=DEV) for r in range(W)]
    out[0] = _off16(out[0])
    rr.ragged_reduce_scatter(plist, bias16, out)
    want = oracle_lib.ragged_reduce_scatter([gu.bits(p) for p in plist], gu.bits(bias), W)
    for r in range(W):
        assert np.array_equal(gu.bits(out[r]), want[r]), r
    # gated, with the gate rows at a 16-modulo-32 address
    gate = _off16(wl.normal_bf16((S, C), 78, 1.0, DEV))
    bounds = wl.segment_bounds(T, S, 79)
    x_full = wl.normal_bf16((T, C), 80, 1.0, DEV)
    x = [v.clone() for v in rr.split_rows(x_full, part.token_starts)]
    x_bits = [gu.bits(v) for v in x]
    rr.ragged_reduce_scatter_gated(plist, bias16, gate, bounds, x)
    want_g = oracle_lib.reduce_scatter_gated([gu.bits(p) for p in plist], gu.bits(bias),
                                             gu.bits(gate), bounds, x_bits, W)
    for r in range(W):
        assert np.array_equal(gu.bits(x[r]), want_g[r]), r
    # all-gather of the reduce-scatter rows into outputs, one of them 16 modulo 32
    outs = [torch.empty((T, C), dtype=torch.bfloat16, device=DEV) for _ in range(W)]
    outs[5] = _off16(outs[5])
    for variant in (0, rr.H3_VARIANT_BULK):
        for o in outs:
            o.zero_()
        rr.ragged_all_gather(out, outs, variant=variant)
        want_a = oracle_lib.ragged_all_gather([gu.bits(v) for v in out], W)
        for j in range(W):
            assert np.array_equal(gu.bits(outs[j]), want_a[j]), (variant, j)


def test_rank_calls_with_16_byte_aligned_peer_buffers():
    """One rank per GPU: a peer's buffer (here a local one standing in for it)
    at 16 modulo 32 bytes; each rank's share equals the one-GPU call's."""
    T, P, H, D, W = 300, 3, 56, 128, 4
    part = rr.partition(T, H, W)
    full = wl.random_bits((T, P, H, D), 91, DEV)
    send = [t.clone() for t in rr.split_rows(full, part.token_starts)]
    send[2] = _off16(send[2])
    ref = rr.alloc_head_side(T, P, H, D, W, DEV)
    rr.seq_to_head(send, ref)
    ref[1] = _off16(ref[1])
    for k in range(W):
        mine = torch.empty_like(ref[k])
        rr.seq_to_head_rank(send, mine, k, n_heads=H)
        assert gu.same_bits(mine, ref[k]), k
        rows = torch.empty_like(send[k])
        rr.head_to_seq_rank(ref, rows, k, n_tokens=T)
        assert gu.same_bits(rows, send[k]), k
    C = 2048
    parts = [wl.normal_bf16((T, C), 92 + r, 0.5, DEV) for r in range(W)]
    parts[3] = _off16(parts[3])
    red = rr.alloc_reduce_outputs(T, C, W, DEV)[1]
    rr.ragged_reduce_scatter(parts, None, red)
    for k in range(W):
        mine = torch.empty_like(red[k])
        rr.ragged_reduce_scatter_rank(parts, None, mine, k, n_tokens=T)
        assert gu.same_bits(mine, red[k]), k


def test_staged_relayouts_with_a_16_byte_aligned_window(oracle_lib):
    """The staged calls through a window buffer at 16 modulo 32 bytes (its
    kernels fall back to 16-byte vectors) equal the oracle."""
    T, P, H, D, W = 300, 3, 56, 128, 4
    part = rr.partition(T, H, W)
    full = wl.random_bits((T, P, H, D), 95, DEV)
    send = rr.split_rows(full, part.token_starts)
    window = _off16(torch.zeros(37 * H * D * 2, dtype=torch.uint8, device=DEV))
    heads = rr.alloc_head_side(T, P, H, D, W, DEV)
    rr.seq_to_head_staged(send, heads, window)
    want = oracle_lib.seq_to_head([gu.bits(s) for s in send], T, P, H, D, W)
    for j in range(W):
        assert np.array_equal(gu.bits(heads[j]), want[j]), j
    back_full, back = rr.alloc_seq_side(T, P, H, D, W, DEV)
    rr.head_to_seq_staged(heads, back, window)
    assert gu.same_bits(back_full, full)
