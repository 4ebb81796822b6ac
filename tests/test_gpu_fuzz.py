"""Seeded random configurations of every entry point against the oracle.

Each case draws its own shape (tokens, planes, heads, head width, world size,
columns, segments), layout, window and kernel variant, and compares the GPU
result with the oracle bit for bit (NaN as "both NaN" where random bit
patterns feed the arithmetic)."""
import numpy as np
import pytest
import torch

import ragged_reduce_b200 as rr
import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

DEV = "cuda"
N_CASES = 40


def _draw_relayout(rng):
    W = int(rng.integers(1, 13))
    H = int(rng.integers(W, max(W + 1, 72)))
    D = int(rng.choice([8, 16, 64, 128, 256]))
    P = int(rng.integers(1, 5))
    T = int(rng.integers(W, 700))
    return T, P, H, D, W


@pytest.mark.parametrize("case", range(N_CASES))
def test_fuzz_relayout(oracle_lib, case):
    rng = np.random.default_rng(1000 + case)
    T, P, H, D, W = _draw_relayout(rng)
    layout = int(rng.integers(0, 4))
    spm, hpm = bool(layout & 1), bool(layout & 2)
    part = rr.partition(T, H, W)
    if spm:
        send = [wl.random_bits((P, part.tokens(r), H, D), case * 97 + r, DEV) for r in range(W)]
    else:
        full = wl.random_bits((T, P, H, D), case * 97, DEV)
        send = rr.split_rows(full, part.token_starts)
    shape = (lambda j: (P, T, part.heads(j), D)) if hpm else (lambda j: (T, P, part.heads(j), D))
    heads = [torch.empty(shape(j), dtype=torch.bfloat16, device=DEV) for j in range(W)]
    plane = max(part.tokens(0) * H * D * 2, T * part.heads(0) * D * 2)
    smallest = max(H * D * 2, W * part.heads(0) * D * 2)  # one token of every rank
    # no window, a whole plane, more than a plane, or less than a plane (token chunks)
    window = int(rng.choice([0, plane, plane * P, int(rng.integers(smallest, plane + 1))]))
    # half the windowed cases cut the window into token ranges of every plane,
    # which needs room for one token of every plane
    tok = window > 0 and bool(rng.integers(0, 2))
    if tok:
        window = max(window, P * smallest)
    variant = int(rng.choice([0, rr.H3_VARIANT_VECTOR]))
    kw = dict(window_bytes=window, token_chunks=tok)
    info = rr.seq_to_head_layout(send, heads, layout, variant=variant, **kw)
    assert info["launches"] == rr.relayout_chunk_plan(T, P, H, D, W, window, token_chunks=tok)[1]
    want = oracle_lib.relayout_layout([gu.bits(s) for s in send], T, P, H, D, W, True, spm, hpm)
    for j in range(W):
        assert np.array_equal(gu.bits(heads[j]), want[j]), (T, P, H, D, W, layout, tok, j)
    back = [torch.empty_like(s) for s in send]
    rr.head_to_seq_layout(heads, back, layout, variant=variant, **kw)
    for r in range(W):
        assert gu.same_bits(back[r], send[r]), (T, P, H, D, W, layout, tok, r)
    if layout == 0 and H * D * 2 * 4 + 128 <= 227 * 1024:  # four row stages fit
        bulk = [torch.empty_like(h) for h in heads]
        rr.seq_to_head(send, bulk, variant=rr.H3_VARIANT_BULK, **kw)
        for j in range(W):
            assert gu.same_bits(bulk[j], heads[j])
    if layout == 0:
        # one rank's shares (one rank per GPU) under the same window
        k = int(rng.integers(0, W))
        mine = torch.empty_like(heads[k])
        rr.seq_to_head_rank(send, mine, k, n_heads=H, **kw)
        assert gu.same_bits(mine, heads[k]), (T, P, H, D, W, window, tok, k)
        rows = torch.empty_like(send[k])
        rr.head_to_seq_rank(heads, rows, k, n_tokens=T, **kw)
        assert gu.same_bits(rows, send[k]), (T, P, H, D, W, window, tok, k)


@pytest.mark.parametrize("case", range(N_CASES // 2))
def test_fuzz_staged(oracle_lib, case):
    rng = np.random.default_rng(2000 + case)
    T, P, H, D, W = _draw_relayout(rng)
    part = rr.partition(T, H, W)
    full = wl.random_bits((T, P, H, D), case * 31, DEV)
    send = rr.split_rows(full, part.token_starts)
    row = H * D * 2
    window = torch.empty(int(rng.integers(row, row * (T + 2))) // 16 * 16 + 16, dtype=torch.uint8,
                         device=DEV)
    heads = rr.alloc_head_side(T, P, H, D, W, DEV)
    rr.seq_to_head_staged(send, heads, window)
    want = oracle_lib.seq_to_head([gu.bits(s) for s in send], T, P, H, D, W)
    for j in range(W):
        assert np.array_equal(gu.bits(heads[j]), want[j]), (T, P, H, D, W, window.numel(), j)
    back_full, back = rr.alloc_seq_side(T, P, H, D, W, DEV)
    rr.head_to_seq_staged(heads, back, window)
    assert gu.same_bits(back_full, full)


@pytest.mark.parametrize("case", range(N_CASES))
def test_fuzz_reduce_gather_gated(oracle_lib, case):
    rng = np.random.default_rng(3000 + case)
    W = int(rng.integers(1, 17))
    T = int(rng.integers(W, 600))
    C = int(rng.integers(1, 160)) * 8
    bits = bool(rng.integers(0, 2))
    with_bias = bool(rng.integers(0, 2))
    if bits:
        partials = wl.random_bits((W, T, C), case, DEV)
        bias = wl.random_bits((C,), case + 1, DEV)
    else:
        rw = wl.ReduceWorkload("f", T=T, C=C, W=W, seed=case)
        partials, bias = wl.partials_and_bias(rw, DEV)
    bias = bias if with_bias else None
    out_full, out = rr.alloc_reduce_outputs(T, C, W, DEV)
    rr.ragged_reduce_scatter(partials, bias, out)
    want = oracle_lib.ragged_reduce_scatter([gu.bits(p) for p in partials],
                                            None if bias is None else gu.bits(bias), W)
    for r in range(W):
        assert gu.nan_aware_equal(gu.bits(out[r]), want[r]).all(), (T, C, W, bits, with_bias, r)
    # all-gather of the reduced rows
    outs = [torch.empty((T, C), dtype=torch.bfloat16, device=DEV) for _ in range(W)]
    rr.ragged_all_gather(out, outs, variant=int(rng.choice([0, rr.H3_VARIANT_BULK])))
    for o in outs:
        assert gu.same_bits(o, out_full)
    # gated, in place on a residual
    S = int(rng.integers(1, min(T, 256) + 1))
    bounds = wl.segment_bounds(T, S, case)
    gate = wl.normal_bf16((S, C), case + 7, 1.0, DEV)
    x_full = wl.normal_bf16((T, C), case + 8, 1.0, DEV)
    x = rr.split_rows(x_full, rr.partition(T, W, W).token_starts)
    x_bits = [gu.bits(v) for v in x]
    rr.ragged_reduce_scatter_gated(partials, bias, gate, bounds, x)
    want = oracle_lib.reduce_scatter_gated([gu.bits(p) for p in partials],
                                           None if bias is None else gu.bits(bias), gu.bits(gate),
                                           bounds, x_bits, W)
    for r in range(W):
        assert gu.nan_aware_equal(gu.bits(x[r]), want[r]).all(), (T, C, W, S, r)
