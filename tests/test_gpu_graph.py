"""The path's calls inside a captured CUDA graph.

Every call enqueues its kernels on the caller's stream and does nothing that
breaks stream capture once a first, eager call has run (per-device caches,
shared-memory opt-in).  A whole step -- seq->head in token chunks, head->seq
one plane per launch, reduce-scatter, all-gather, gated reduce-scatter -- is
captured once, the inputs are overwritten in place, and each replay must give
the oracle's results for the new inputs."""
import numpy as np
import pytest
import torch

import ragged_reduce_b200 as rr
import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

DEV = "cuda"


def test_step_replays_from_a_cuda_graph(oracle_lib):
    T, P, H, D, W, C, S = 600, 3, 56, 128, 6, 1024, 4
    part = rr.partition(T, H, W)
    x = wl.random_bits((T, P, H, D), 1, DEV)
    send = rr.split_rows(x, part.token_starts)
    heads = rr.alloc_head_side(T, P, H, D, W, DEV)
    back_full, back = rr.alloc_seq_side(T, P, H, D, W, DEV)
    window = max(part.tokens(0) * H * D * 2, T * part.heads(0) * D * 2)
    partials = wl.normal_bf16((W, T, C), 2, 0.5, DEV)
    bias = wl.normal_bf16((C,), 3, 0.1, DEV)
    red_full, red = rr.alloc_reduce_outputs(T, C, W, DEV)
    gath = [torch.empty((T, C), dtype=torch.bfloat16, device=DEV) for _ in range(W)]
    gate = wl.normal_bf16((S, C), 4, 1.0, DEV)
    bounds = wl.segment_bounds(T, S, 5)
    resid_src = wl.normal_bf16((T, C), 6, 1.0, DEV)
    resid_full = resid_src.clone()
    resid = rr.split_rows(resid_full, rr.partition(T, W, W).token_starts)

    # seq->head with every plane in token chunks, head->seq one plane per
    # launch, then seq->head again in token ranges of every plane into a
    # second set of buffers
    sub = gu.chunk_window("sub", T, H, D, W)
    assert rr.relayout_chunk_plan(T, P, H, D, W, sub)[1] > P
    ranges_window = gu.range_window("half", T, P, H, D, W)
    assert rr.relayout_chunk_plan(T, P, H, D, W, ranges_window, token_chunks=True)[1] > 1
    heads2 = rr.alloc_head_side(T, P, H, D, W, DEV)

    def step():
        rr.seq_to_head(send, heads, window_bytes=sub)
        rr.head_to_seq(heads, back, window_bytes=window)
        rr.seq_to_head(send, heads2, window_bytes=ranges_window, token_chunks=True)
        rr.ragged_reduce_scatter(partials, bias, red)
        rr.ragged_all_gather(red, gath)
        resid_full.copy_(resid_src)
        rr.ragged_reduce_scatter_gated(partials, bias, gate, bounds, resid)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()  # eager first call: caches and opt-ins are set outside capture
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()

    for round_ in range(3):
        x.copy_(wl.random_bits((T, P, H, D), 10 + round_, DEV))
        partials.copy_(wl.normal_bf16((W, T, C), 20 + round_, 0.5, DEV))
        graph.replay()
        torch.cuda.synchronize()
        want = oracle_lib.seq_to_head([gu.bits(s) for s in send], T, P, H, D, W)
        for j in range(W):
            assert np.array_equal(gu.bits(heads[j]), want[j]), (round_, j)
            assert gu.same_bits(heads2[j], heads[j]), (round_, j)
        assert gu.same_bits(back_full, x)
        want_red = oracle_lib.ragged_reduce_scatter([gu.bits(p) for p in partials.unbind(0)],
                                                    gu.bits(bias), W)
        for r in range(W):
            assert np.array_equal(gu.bits(red[r]), want_red[r]), (round_, r)
        for g in gath:
            assert gu.same_bits(g, red_full)
        want_g = oracle_lib.reduce_scatter_gated(
            [gu.bits(p) for p in partials.unbind(0)], gu.bits(bias), gu.bits(gate), bounds,
            [gu.bits(v) for v in rr.split_rows(resid_src, rr.partition(T, W, W).token_starts)], W)
        for r in range(W):
            assert np.array_equal(gu.bits(resid[r]), want_g[r]), (round_, r)
    del graph
