"""GPU parity of the ragged reduce-scatter against the CPU oracle (bit-exact).

The contract is bit-exact under the fixed rank order: the kernel and the
oracle both widen BF16 exactly, add in binary32 in rank order 0..W-1 from
partial 0, add the bias once, and round to nearest even.  NaN results are
compared as "both NaN" (the NaN payload is not part of the contract).
"""
import numpy as np
import pytest
import torch

import ragged_reduce_b200 as rr
import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _run(partials, bias, T, C, W):
    out_full, out = rr.alloc_reduce_outputs(T, C, W, DEV)
    info = rr.ragged_reduce_scatter(partials, bias, out)
    return out_full, out, info


@pytest.mark.parametrize("T,C,W", [
    (1000, 7168, 6), (1024, 7168, 8), (333, 7168, 3), (64, 7168, 1), (97, 2048, 2),
    (50, 4104, 4), (129, 8, 5), (200, 1024, 7), (90, 512, 9), (70, 256, 16), (64, 64, 64),
])
@pytest.mark.parametrize("with_bias", [True, False])
def test_reduce_matches_oracle(oracle_lib, T, C, W, with_bias):
    w = wl.ReduceWorkload("t", T=T, C=C, W=W, seed=T + C + W)
    partials, bias = wl.partials_and_bias(w, DEV)
    if not with_bias:
        bias = None
    out_full, out, info = _run(partials, bias, T, C, W)
    assert info["launches"] == 1
    want = oracle_lib.ragged_reduce_scatter([gu.bits(p) for p in partials],
                                            None if bias is None else gu.bits(bias), W)
    for r in range(W):
        got = gu.bits(out[r])
        bad = np.flatnonzero(got != want[r])
        assert bad.size == 0, f"rank {r}: {bad.size} mismatches"


def test_reduce_random_bit_patterns(oracle_lib):
    """Inf, NaN, subnormals and signed zeros in every position."""
    T, C, W = 300, 1024, 5
    partials = wl.random_bits((W, T, C), 31, DEV)
    bias = wl.random_bits((C,), 32, DEV)
    _, out, _ = _run(partials, bias, T, C, W)
    want = oracle_lib.ragged_reduce_scatter([gu.bits(p) for p in partials], gu.bits(bias), W)
    for r in range(W):
        ok = gu.nan_aware_equal(gu.bits(out[r]), want[r])
        assert ok.all(), f"rank {r}: {np.count_nonzero(~ok)} mismatches"


def test_reduce_zero_partials_give_bias():
    T, C, W = 77, 7168, 4
    partials = torch.zeros((W, T, C), dtype=torch.bfloat16, device=DEV)
    bias = wl.normal_bf16((C,), 8, 0.1, DEV)
    bias[bias == 0] = 1.0  # +0 + -0 is +0; keep the bias non-zero
    out_full, _, _ = _run(partials, bias, T, C, W)
    assert gu.same_bits(out_full, bias.expand(T, C))


def test_reduce_split_gemm_integer():
    """Sharded partials of an integer GEMM sum to the unsharded result plus the
    bias once ("Distributed H3 Execution", "Partition Contract")."""
    rng = np.random.default_rng(41)
    T, K, C, W = 1000, 12, 7168, 6
    X = rng.integers(-4, 5, size=(T, K))
    Wt = rng.integers(-4, 5, size=(C, K))
    b = rng.integers(-8, 9, size=C)
    kq, km = K // W, K % W
    ks = [i * kq + min(i, km) for i in range(W + 1)]
    parts = [torch.from_numpy((X[:, ks[w]:ks[w + 1]] @ Wt[:, ks[w]:ks[w + 1]].T).astype(np.float32))
             .to(torch.bfloat16).to(DEV) for w in range(W)]
    full = torch.from_numpy((X @ Wt.T + b[None, :]).astype(np.float32)).to(torch.bfloat16)
    bias = torch.from_numpy(b.astype(np.float32)).to(torch.bfloat16).to(DEV)
    out_full, _, _ = _run(parts, bias, T, C, W)
    assert gu.same_bits(out_full.cpu(), full)


def test_reduce_guard_bands():
    T, C, W = 1000, 7168, 6
    w = wl.ReduceWorkload("t", T=T, C=C, W=W, seed=5)
    partials, bias = wl.partials_and_bias(w, DEV)
    part = rr.partition(T, W, W)
    bufs, outs = [], []
    for r in range(W):
        buf, o = gu.guarded((part.tokens(r), C), DEV)
        bufs.append(buf)
        outs.append(o)
    rr.ragged_reduce_scatter(partials, bias, outs)
    assert all(gu.guards_intact(b) for b in bufs)


def test_full_reduce_scatter_64k_w8(oracle_lib):
    w = wl.RS_64K_W8
    partials, bias = wl.partials_and_bias(w, DEV)
    out_full, out, info = _run(partials, bias, w.T, w.C, w.W)
    assert info["launches"] == 1
    part = rr.partition(w.T, w.W, w.W)
    # sampled rows through the oracle, including every rank's first and last row
    rng = np.random.default_rng(w.seed)
    rows = np.unique(np.concatenate([rng.integers(0, w.T, 192),
                                     part.token_starts[:-1], part.token_starts[1:] - 1]))
    rows_t = torch.from_numpy(rows).to(DEV)
    sub = [gu.bits(partials[k].index_select(0, rows_t)) for k in range(w.W)]
    want = oracle_lib.reduce_rows(sub, gu.bits(bias))
    got = gu.bits(out_full.index_select(0, rows_t))
    assert np.array_equal(got, want)
    # every element against torch's binary32 elementwise adds in the same order
    # (a third opinion at full size)
    acc = partials[0].float()
    for k in range(1, w.W):
        acc += partials[k].float()
    acc += bias.float()
    assert gu.same_bits(out_full, acc.to(torch.bfloat16))
    # rows land in their rank's buffer
    for r in range(w.W):
        assert out[r].data_ptr() == out_full[int(part.token_starts[r])].data_ptr()


def test_prepared_reduce_scatter(oracle_lib):
    T, C, W = 500, 7168, 6
    w = wl.ReduceWorkload("p", T=T, C=C, W=W, seed=12)
    partials, bias = wl.partials_and_bias(w, DEV)
    out_full, out = rr.alloc_reduce_outputs(T, C, W, DEV)
    call = rr.prepare_ragged_reduce_scatter(list(partials.unbind(0)), bias, out)
    for round_ in range(2):
        partials.copy_(wl.normal_bf16((W, T, C), 40 + round_, 0.5, DEV))
        call()
        want = oracle_lib.ragged_reduce_scatter([gu.bits(p) for p in partials.unbind(0)],
                                                gu.bits(bias), W)
        for r in range(W):
            assert np.array_equal(gu.bits(out[r]), want[r])


@pytest.mark.parametrize("W", range(1, 9))
@pytest.mark.parametrize("C", [1024, 1040])
def test_every_compiled_width_matches_oracle(oracle_lib, W, C):
    """Both vector widths for every compile-time W: C = 1024 gives 32-byte
    aligned rows (the 32-byte kernels), C = 1040 rows of 2,080 bytes (the
    16-byte kernels); plain and gated reduce-scatter."""
    T = 257 + W
    w = wl.ReduceWorkload("w", T=T, C=C, W=W, seed=W * 31 + C)
    partials, bias = wl.partials_and_bias(w, DEV)
    out_full, out, info = _run(partials, bias, T, C, W)
    want = oracle_lib.ragged_reduce_scatter([gu.bits(p) for p in partials], gu.bits(bias), W)
    for r in range(W):
        assert np.array_equal(gu.bits(out[r]), want[r]), (W, C, r)
    S = 3
    gate = wl.normal_bf16((S, C), W + 5, 1.0, DEV)
    bounds = wl.segment_bounds(T, S, W)
    x_full = wl.normal_bf16((T, C), W + 6, 1.0, DEV)
    part = rr.partition(T, W, W)
    x = [v.clone() for v in rr.split_rows(x_full, part.token_starts)]
    rr.ragged_reduce_scatter_gated(partials, bias, gate, bounds, x)
    want_g = oracle_lib.reduce_scatter_gated([gu.bits(p) for p in partials], gu.bits(bias),
                                             gu.bits(gate), bounds,
                                             [gu.bits(v) for v in rr.split_rows(x_full, part.token_starts)], W)
    for r in range(W):
        assert np.array_equal(gu.bits(x[r]), want_g[r]), (W, C, r)
