"""GPU parity of the reduce-scatter fused with per-segment residual gating."""
import numpy as np
import pytest
import torch

import ragged_reduce_b200 as rr
import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _inputs(T, C, W, S, seed, bits=False):
    rw = wl.ReduceWorkload("g", T=T, C=C, W=W, seed=seed)
    if bits:
        partials = wl.random_bits((W, T, C), seed, DEV)
        bias = wl.random_bits((C,), seed + 1, DEV)
        gate = wl.random_bits((S, C), seed + 2, DEV)
    else:
        partials, bias = wl.partials_and_bias(rw, DEV)
        gate = wl.normal_bf16((S, C), seed + 2, 1.0, DEV)
    bounds = wl.segment_bounds(T, S, seed)
    part = rr.partition(T, W, W)
    x_full = wl.normal_bf16((T, C), seed + 3, 1.0, DEV)
    return partials, bias, gate, bounds, x_full, rr.split_rows(x_full, part.token_starts)


@pytest.mark.parametrize("T,C,W,S", [(1000, 7168, 6, 8), (1024, 7168, 2, 3), (333, 7168, 3, 16),
                                     (97, 2048, 8, 5), (64, 64, 64, 1), (90, 512, 9, 7),
                                     (300, 1024, 5, 256)])
@pytest.mark.parametrize("in_place", [False, True])
@pytest.mark.parametrize("with_bias", [True, False])
def test_gated_matches_oracle(oracle_lib, T, C, W, S, in_place, with_bias):
    partials, bias, gate, bounds, x_full, x = _inputs(T, C, W, S, T + W + S)
    if not with_bias:
        bias = None  # the bias is optional, as in the plain reduce-scatter
    x_bits = [gu.bits(v) for v in x]
    if in_place:
        out = x
        info = rr.ragged_reduce_scatter_gated(partials, bias, gate, bounds, x)
    else:
        out_full, out = rr.alloc_reduce_outputs(T, C, W, DEV)
        info = rr.ragged_reduce_scatter_gated(partials, bias, gate, bounds, x, out)
    assert info["launches"] == 1
    want = oracle_lib.reduce_scatter_gated([gu.bits(p) for p in partials],
                                           gu.bits(bias) if with_bias else None,
                                           gu.bits(gate), bounds, x_bits, W)
    for r in range(W):
        assert np.array_equal(gu.bits(out[r]), want[r]), f"rank {r}"


def test_gated_equals_reduce_scatter_then_gating_full_size(oracle_lib):
    """The 64k x 7168 x 8 workload, 16 segments: every element against the
    unfused composition (torch binary32 gating on the plain reduce-scatter
    output), and sampled rows -- every rank and segment boundary among them --
    through the oracle."""
    T, C, W, S = 65536, 7168, 8, 16
    partials, bias, gate, bounds, x_full, x = _inputs(T, C, W, S, 4)
    red_full, red = rr.alloc_reduce_outputs(T, C, W, DEV)
    rr.ragged_reduce_scatter(partials, bias, red)
    seg = torch.from_numpy(np.searchsorted(bounds, np.arange(T), side="right") - 1).to(DEV)
    want = (x_full.float() + gate.float()[seg] * red_full.float()).to(torch.bfloat16)
    out_full, out = rr.alloc_reduce_outputs(T, C, W, DEV)
    rr.ragged_reduce_scatter_gated(partials, bias, gate, bounds, x, out)
    assert gu.same_bits(out_full, want)
    # sampled rows through the oracle: each sampled row becomes a segment of
    # its own carrying its original gate row, the rows split over W ranks
    ts = rr.partition(T, W, W).token_starts
    rng = np.random.default_rng(44)
    b = np.asarray(bounds)
    rows = np.unique(np.concatenate([rng.integers(0, T, 160), ts[:-1], ts[1:] - 1, b[:-1], b[1:] - 1]))
    rows_t = torch.from_numpy(rows).to(DEV)
    sub_parts = [gu.bits(partials[k].index_select(0, rows_t)) for k in range(W)]
    sub_gate = gu.bits(gate.index_select(0, seg.index_select(0, rows_t)))
    sub_bounds = np.arange(len(rows) + 1, dtype=np.int64)
    sub_x = gu.bits(x_full.index_select(0, rows_t))
    sts = oracle_lib.partition_range(len(rows), W)
    got = oracle_lib.reduce_scatter_gated(sub_parts, gu.bits(bias), sub_gate, sub_bounds,
                                          [sub_x[sts[r]:sts[r + 1]] for r in range(W)], W)
    assert np.array_equal(np.concatenate(got), gu.bits(out_full.index_select(0, rows_t)))


def test_gated_random_bit_patterns(oracle_lib):
    T, C, W, S = 200, 1024, 5, 4
    partials, bias, gate, bounds, x_full, x = _inputs(T, C, W, S, 77, bits=True)
    out_full, out = rr.alloc_reduce_outputs(T, C, W, DEV)
    rr.ragged_reduce_scatter_gated(partials, bias, gate, bounds, x, out)
    want = oracle_lib.reduce_scatter_gated([gu.bits(p) for p in partials], gu.bits(bias),
                                           gu.bits(gate), bounds, [gu.bits(v) for v in x], W)
    for r in range(W):
        ok = gu.nan_aware_equal(gu.bits(out[r]), want[r])
        assert ok.all(), f"rank {r}: {np.count_nonzero(~ok)} mismatches"


def test_gated_rejects_bad_segments_and_partial_overlap():
    T, C, W, S = 100, 512, 4, 3
    partials, bias, gate, bounds, x_full, x = _inputs(T, C, W, S, 5)
    out_full, out = rr.alloc_reduce_outputs(T, C, W, DEV)
    with pytest.raises(rr.H3Error) as e:
        rr.ragged_reduce_scatter_gated(partials, bias, gate, [0, 50, 50, 100], x, out)
    assert e.value.status == 1
    shifted = [x_full[8:33]] + out[1:]  # out[0] partly overlaps x[0]
    with pytest.raises(rr.H3Error) as e:
        rr.ragged_reduce_scatter_gated(partials, bias, gate, bounds, x, shifted)
    assert e.value.status == 1
