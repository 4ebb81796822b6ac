"""GPU parity of the ragged all-gather against the CPU oracle (bit-exact)."""
import numpy as np
import pytest
import torch

import ragged_reduce_b200 as rr
import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _blocks(T, C, W, seed):
    full = wl.random_bits((T, C), seed, DEV)
    part = rr.partition(T, W, W)
    return full, rr.split_rows(full, part.token_starts)


@pytest.mark.parametrize("T,C,W", [(1000, 7168, 6), (97, 8, 8), (64, 4104, 4), (33, 24, 1),
                                   (200, 7168, 8), (90, 18000, 3), (64, 64, 64), (7, 7168, 7)])
def test_all_gather_matches_oracle(oracle_lib, T, C, W):
    full, blocks = _blocks(T, C, W, T + C + W)
    outs = [torch.empty((T, C), dtype=torch.bfloat16, device=DEV) for _ in range(W)]
    info = rr.ragged_all_gather(blocks, outs)
    assert info["launches"] == 1 and info["variant"] == rr.H3_VARIANT_GATHER
    want = oracle_lib.ragged_all_gather([gu.bits(b) for b in blocks], W)
    for j in range(W):
        assert np.array_equal(gu.bits(outs[j]), want[j]), f"rank {j}"


@pytest.mark.parametrize("T,C,W", [(1000, 7168, 6), (97, 8, 8), (64, 4104, 4), (33, 24, 1), (7, 7168, 7)])
@pytest.mark.parametrize("variant", [rr.H3_VARIANT_VECTOR, rr.H3_VARIANT_BULK])
def test_all_gather_forced_variant(oracle_lib, T, C, W, variant):
    full, blocks = _blocks(T, C, W, 3 * T + W)
    bufs, outs = [], []
    for _ in range(W):
        b, o = gu.guarded((T, C), DEV)
        bufs.append(b)
        outs.append(o)
    rr.bulk_wait_timeouts(reset=True)
    info = rr.ragged_all_gather(blocks, outs, variant=variant)
    assert info["variant"] == (rr.H3_VARIANT_BULK if variant == rr.H3_VARIANT_BULK else rr.H3_VARIANT_GATHER)
    want = oracle_lib.ragged_all_gather([gu.bits(b) for b in blocks], W)
    for j in range(W):
        assert np.array_equal(gu.bits(outs[j]), want[j]), f"rank {j}"
    assert all(gu.guards_intact(b) for b in bufs)
    assert rr.bulk_wait_timeouts() == 0


@pytest.mark.parametrize("ctas_per_sm", [0, 1])
def test_all_gather_bulk_row_groups_and_capped_grid(oracle_lib, ctas_per_sm):
    """The bulk all-gather launches one warp per four rows; capped at one CTA
    per SM every CTA walks several row groups and refills its stages.  Rows
    of 36,000 bytes: four stages fit in shared memory."""
    for T, C, W in [(3001, 7168, 8), (301, 18000, 3)]:
        full, blocks = _blocks(T, C, W, 11 * T + W + ctas_per_sm)
        outs = [torch.empty((T, C), dtype=torch.bfloat16, device=DEV) for _ in range(W)]
        rr.bulk_wait_timeouts(reset=True)
        info = rr.ragged_all_gather(blocks, outs, variant=rr.H3_VARIANT_BULK, ctas_per_sm=ctas_per_sm)
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        groups = (T + 3) // 4
        assert info["variant"] == rr.H3_VARIANT_BULK and info["block"] == 32
        assert info["grid"] == (groups if not ctas_per_sm else min(groups, ctas_per_sm * sms))
        want = oracle_lib.ragged_all_gather([gu.bits(b) for b in blocks], W)
        for j in range(W):
            assert np.array_equal(gu.bits(outs[j]), want[j]), f"rank {j}"
        assert rr.bulk_wait_timeouts() == 0


def test_all_gather_bulk_rejects_wide_rows():
    T, C, W = 16, 30000, 2  # 60,000-byte rows: four stages do not fit
    full, blocks = _blocks(T, C, W, 1)
    outs = [torch.empty((T, C), dtype=torch.bfloat16, device=DEV) for _ in range(W)]
    with pytest.raises(rr.H3Error) as e:
        rr.ragged_all_gather(blocks, outs, variant=rr.H3_VARIANT_BULK)
    assert e.value.status == 5


def test_all_gather_guard_bands_and_separate_blocks(oracle_lib):
    T, C, W = 500, 7168, 6
    part = rr.partition(T, W, W)
    blocks = [wl.random_bits((part.tokens(r), C), 40 + r, DEV) for r in range(W)]
    bufs, outs = [], []
    for _ in range(W):
        b, o = gu.guarded((T, C), DEV)
        bufs.append(b)
        outs.append(o)
    rr.ragged_all_gather(blocks, outs)
    assert all(gu.guards_intact(b) for b in bufs)
    want = oracle_lib.ragged_all_gather([gu.bits(b) for b in blocks], W)
    for j in range(W):
        assert np.array_equal(gu.bits(outs[j]), want[j])


def test_reduce_scatter_then_all_gather_is_unsharded_gemm():
    """Tensor mode end to end: sharded integer-GEMM partials, ragged
    reduce-scatter with the bias once, ragged all-gather: every rank holds
    X W^T + b ("Distributed H3 Execution", "Partition Contract")."""
    rng = np.random.default_rng(43)
    T, K, C, W = 1000, 12, 7168, 6
    X = rng.integers(-4, 5, size=(T, K))
    Wt = rng.integers(-4, 5, size=(C, K))
    b = rng.integers(-8, 9, size=C)
    ks = [i * (K // W) + min(i, K % W) for i in range(W + 1)]
    parts = [torch.from_numpy((X[:, ks[w]:ks[w + 1]] @ Wt[:, ks[w]:ks[w + 1]].T).astype(np.float32))
             .to(torch.bfloat16).to(DEV) for w in range(W)]
    bias = torch.from_numpy(b.astype(np.float32)).to(torch.bfloat16).to(DEV)
    red_full, red = rr.alloc_reduce_outputs(T, C, W, DEV)
    rr.ragged_reduce_scatter(parts, bias, red)
    outs = [torch.empty((T, C), dtype=torch.bfloat16, device=DEV) for _ in range(W)]
    rr.ragged_all_gather(red, outs)
    want = torch.from_numpy((X @ Wt.T + b[None, :]).astype(np.float32)).to(torch.bfloat16)
    for o in outs:
        assert gu.same_bits(o.cpu(), want)


def test_full_all_gather_64k_w8():
    """Every output equals the full [65536, 7168] rows, with the register
    kernel and with the bulk (TMA) kernel."""
    T, C, W = 65536, 7168, 8
    full, blocks = _blocks(T, C, W, 4)
    outs = [torch.empty((T, C), dtype=torch.bfloat16, device=DEV) for _ in range(W)]
    rr.bulk_wait_timeouts(reset=True)
    for variant in (0, rr.H3_VARIANT_BULK):
        for o in outs:
            o.zero_()
        rr.ragged_all_gather(blocks, outs, variant=variant)
        for o in outs:
            assert gu.same_bits(o, full), variant
    assert rr.bulk_wait_timeouts() == 0
