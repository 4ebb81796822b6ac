"""GPU parity of the Ulysses relayouts against the CPU oracle (bit-exact).

Small shapes are compared element by element with the oracle's full loops;
full-size workloads are compared on sampled elements through the oracle's
gather map, plus properties that hold at any size (round trip, torch slicing).
"""
import numpy as np
import pytest
import torch

import ragged_reduce_b200 as rr
import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _seq_inputs(T, P, H, D, W, seed, kind="bits"):
    if kind == "bits":
        full = wl.random_bits((T, P, H, D), seed, DEV)
    else:
        full = wl.normal_bf16((T, P, H, D), seed, 1.0, DEV)
    part = rr.partition(T, H, W)
    return full, rr.split_rows(full, part.token_starts), part


# T, P, H, D, W: ragged tokens and heads, several CTAs' worth of rows, every
# kernel template (1..8 vectors per thread, two-row and one-row), the generic
# kernel (rows wider than 1024 vectors), narrow 16-byte heads, one head per
# rank, one token per rank.
SMALL = [
    (1024, 3, 56, 128, 2),
    (1000, 3, 56, 128, 6),
    (777, 4, 56, 128, 8),
    (513, 1, 56, 128, 4),
    (100, 3, 56, 128, 1),
    (64, 3, 56, 128, 56),
    (9, 3, 56, 128, 9),
    (130, 2, 7, 64, 3),
    (50, 3, 5, 8, 5),
    (301, 2, 16, 64, 5),
    (40, 3, 24, 128, 7),
    (20, 2, 300, 128, 7),
    (33, 3, 56, 256, 4),
    (7, 4, 56, 128, 7),
]


@pytest.mark.parametrize("T,P,H,D,W", SMALL)
@pytest.mark.parametrize("window", [0, "plane"])
def test_relayout_matches_oracle(oracle_lib, T, P, H, D, W, window):
    full, send, part = _seq_inputs(T, P, H, D, W, seed=T * 31 + W)
    if window == "plane":
        window = max(part.tokens(0) * H * D * 2, T * part.heads(0) * D * 2)
    recv = rr.alloc_head_side(T, P, H, D, W, DEV)
    info = rr.seq_to_head(send, recv, window_bytes=window)
    assert info["launches"] == (P if window else 1)
    want = oracle_lib.seq_to_head([gu.bits(s) for s in send], T, P, H, D, W)
    for j in range(W):
        assert np.array_equal(gu.bits(recv[j]), want[j]), f"seq->head rank {j}"
    back_full, back = rr.alloc_seq_side(T, P, H, D, W, DEV)
    info = rr.head_to_seq(recv, back, window_bytes=window)
    assert info["launches"] == (P if window else 1)
    want_back = oracle_lib.head_to_seq(want, T, P, H, D, W)
    for r in range(W):
        assert np.array_equal(gu.bits(back[r]), want_back[r]), f"head->seq rank {r}"
    assert gu.same_bits(back_full, full)  # round trip


# every kernel family forced through the _ex entry points, both directions
VARIANT_SHAPES = [
    (1000, 3, 56, 128, 6),
    (777, 4, 56, 128, 8),
    (513, 2, 56, 128, 4),
    (64, 3, 56, 128, 2),
    (100, 3, 56, 128, 1),
    (9, 3, 56, 128, 9),
    (130, 2, 7, 64, 3),
    (50, 3, 5, 8, 5),
    (40, 3, 24, 128, 7),
]


@pytest.mark.parametrize("T,P,H,D,W", VARIANT_SHAPES)
@pytest.mark.parametrize("variant", [rr.H3_VARIANT_VECTOR, rr.H3_VARIANT_BULK])
def test_forced_variant_matches_oracle(oracle_lib, T, P, H, D, W, variant):
    full, send, part = _seq_inputs(T, P, H, D, W, seed=T * 7 + W + variant)
    recv = rr.alloc_head_side(T, P, H, D, W, DEV)
    rr.bulk_wait_timeouts(reset=True)
    info = rr.seq_to_head(send, recv, variant=variant)
    assert info["variant"] == variant
    want = oracle_lib.seq_to_head([gu.bits(s) for s in send], T, P, H, D, W)
    for j in range(W):
        assert np.array_equal(gu.bits(recv[j]), want[j]), f"seq->head rank {j}"
    back_full, back = rr.alloc_seq_side(T, P, H, D, W, DEV)
    plane = max(part.tokens(0) * H * D * 2, T * part.heads(0) * D * 2)
    info = rr.head_to_seq(recv, back, variant=variant, window_bytes=plane)
    assert info["variant"] == variant and info["launches"] == P
    assert gu.same_bits(back_full, full)
    assert rr.bulk_wait_timeouts() == 0


def test_bulk_row_width_limit(oracle_lib):
    """A bulk CTA stages four rows: a 28,672-byte row (D=256) fits and
    matches the oracle; a 114,688-byte row (D=1024) does not fit in shared
    memory and is refused, while the default call still runs it."""
    T, P, H, D, W = 33, 3, 56, 256, 4
    full, send, part = _seq_inputs(T, P, H, D, W, seed=1)
    recv = rr.alloc_head_side(T, P, H, D, W, DEV)
    info = rr.seq_to_head(send, recv, variant=rr.H3_VARIANT_BULK)
    assert info["variant"] == rr.H3_VARIANT_BULK
    want = oracle_lib.seq_to_head([gu.bits(x) for x in send], T, P, H, D, W)
    for j in range(W):
        assert np.array_equal(gu.bits(recv[j]), want[j]), j

    T, P, H, D, W = 9, 2, 56, 1024, 4
    full, send, part = _seq_inputs(T, P, H, D, W, seed=2)
    recv = rr.alloc_head_side(T, P, H, D, W, DEV)
    with pytest.raises(rr.H3Error) as e:
        rr.seq_to_head(send, recv, variant=rr.H3_VARIANT_BULK)
    assert e.value.status == 5  # H3_ERR_UNSUPPORTED
    info = rr.seq_to_head(send, recv)  # the default takes the register kernels
    assert info["variant"] != rr.H3_VARIANT_BULK
    want = oracle_lib.seq_to_head([gu.bits(x) for x in send], T, P, H, D, W)
    for j in range(W):
        assert np.array_equal(gu.bits(recv[j]), want[j]), j


def test_bulk_stage_sizes_alternate(oracle_lib):
    """Bulk launches whose shared-memory stages differ in size, in both orders
    (a smaller launch must not shrink what a later, larger one may use)."""
    for T, P, H, D, W in [(40, 3, 24, 128, 3), (64, 3, 56, 128, 2), (40, 3, 24, 128, 3),
                          (64, 3, 56, 128, 4), (130, 2, 7, 64, 3), (64, 3, 56, 128, 2)]:
        full, send, part = _seq_inputs(T, P, H, D, W, seed=T + H + W)
        recv = rr.alloc_head_side(T, P, H, D, W, DEV)
        rr.seq_to_head(send, recv, variant=rr.H3_VARIANT_BULK)
        back_full, back = rr.alloc_seq_side(T, P, H, D, W, DEV)
        rr.head_to_seq(recv, back, variant=rr.H3_VARIANT_BULK)
        assert gu.same_bits(back_full, full)
        want = oracle_lib.seq_to_head([gu.bits(s) for s in send], T, P, H, D, W)
        for j in range(W):
            assert np.array_equal(gu.bits(recv[j]), want[j])


@pytest.mark.parametrize("ctas_per_sm", [0, 1, 3])
def test_bulk_row_groups_and_capped_grid(oracle_lib, ctas_per_sm):
    """The bulk kernel launches one warp per four rows.  A capped grid makes
    every CTA walk several row groups, so each lane refills its stage and
    reuses its barrier (the stage only after its stores have read it); both
    directions, one plane per launch on the way back."""
    T, P, H, D, W = 2003, 3, 56, 128, 6
    full, send, part = _seq_inputs(T, P, H, D, W, seed=97 + ctas_per_sm)
    sms = torch.cuda.get_device_properties(0).multi_processor_count

    def grid(rows):
        groups = (rows + 3) // 4
        return groups if not ctas_per_sm else min(groups, ctas_per_sm * sms)

    recv = rr.alloc_head_side(T, P, H, D, W, DEV)
    rr.bulk_wait_timeouts(reset=True)
    info = rr.seq_to_head(send, recv, variant=rr.H3_VARIANT_BULK, ctas_per_sm=ctas_per_sm)
    assert info["variant"] == rr.H3_VARIANT_BULK and info["block"] == 32
    assert info["grid"] == grid(T * P)
    want = oracle_lib.seq_to_head([gu.bits(s) for s in send], T, P, H, D, W)
    for j in range(W):
        assert np.array_equal(gu.bits(recv[j]), want[j]), f"seq->head rank {j}"
    back_full, back = rr.alloc_seq_side(T, P, H, D, W, DEV)
    plane = max(part.tokens(0) * H * D * 2, T * part.heads(0) * D * 2)
    info = rr.head_to_seq(recv, back, variant=rr.H3_VARIANT_BULK, ctas_per_sm=ctas_per_sm,
                          window_bytes=plane)
    assert info["launches"] == P and info["grid"] == grid(T)
    assert gu.same_bits(back_full, full)
    assert rr.bulk_wait_timeouts() == 0


def test_default_variants():
    """Defaults: the vector kernels in both directions, one CTA per row pair
    (seq->head) or row (head->seq); the bulk kernel only when asked for."""
    for W, want_back in [(2, rr.H3_VARIANT_VECTOR), (4, rr.H3_VARIANT_VECTOR), (6, rr.H3_VARIANT_VECTOR)]:
        T, P, H, D = 300, 3, 56, 128
        full, send, part = _seq_inputs(T, P, H, D, W, seed=W)
        recv = rr.alloc_head_side(T, P, H, D, W, DEV)
        info = rr.seq_to_head(send, recv)
        assert info["variant"] == rr.H3_VARIANT_VECTOR
        assert info["grid"] == (T * P + 1) // 2
        back_full, back = rr.alloc_seq_side(T, P, H, D, W, DEV)
        info = rr.head_to_seq(recv, back)
        assert info["variant"] == want_back and info["grid"] == T * P
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        capped = rr.head_to_seq(recv, back, ctas_per_sm=2)
        assert capped["grid"] == min(2 * sms, T * P)
        assert gu.same_bits(back_full, full)
        assert gu.same_bits(back_full, full)


def test_world_one_identity():
    T, P, H, D = 257, 3, 56, 128
    full = wl.random_bits((T, P, H, D), 5, DEV)
    (recv,) = rr.alloc_head_side(T, P, H, D, 1, DEV)
    rr.seq_to_head([full], [recv])
    assert gu.same_bits(recv, full)
    back = torch.empty_like(full)
    rr.head_to_seq([recv], [back])
    assert gu.same_bits(back, full)


def test_tiny_workload_round_trip(oracle_lib):
    w = wl.TINY_QKV_W2
    full = wl.packed_operand(w, device=DEV)
    bounds = wl.segment_bounds(w.T, w.n_segs, w.seed, w.seg_lengths)
    part = rr.partition(w.T, w.H, w.W, bounds)
    assert [list(b) for b in part.local_bounds] == [[0, 400, 512], [0, 225, 512]]
    send = rr.split_rows(full, part.token_starts)
    recv = rr.alloc_head_side(w.T, w.P, w.H, w.D, w.W, DEV)
    rr.seq_to_head(send, recv)
    want = oracle_lib.seq_to_head([gu.bits(s) for s in send], w.T, w.P, w.H, w.D, w.W)
    for j in range(w.W):
        assert np.array_equal(gu.bits(recv[j]), want[j])
    back_full, back = rr.alloc_seq_side(w.T, w.P, w.H, w.D, w.W, DEV)
    rr.head_to_seq(recv, back)
    assert gu.same_bits(back_full, full)


def test_guard_bands_untouched():
    T, P, H, D, W = 1000, 3, 56, 128, 6
    full, send, part = _seq_inputs(T, P, H, D, W, seed=9)
    bufs, recv = [], []
    for j in range(W):
        b, o = gu.guarded((T, P, part.heads(j), D), DEV)
        bufs.append(b)
        recv.append(o)
    rr.seq_to_head(send, recv)
    assert all(gu.guards_intact(b) for b in bufs)
    sbufs, back = [], []
    for r in range(W):
        b, o = gu.guarded((part.tokens(r), P, H, D), DEV)
        sbufs.append(b)
        back.append(o)
    rr.head_to_seq(recv, back)
    assert all(gu.guards_intact(b) for b in sbufs)
    assert gu.same_bits(torch.cat(back), full)


def test_separate_send_buffers_and_side_stream(oracle_lib):
    """Send buffers in separate allocations, work on a non-default stream."""
    T, P, H, D, W = 600, 4, 56, 128, 4
    part = rr.partition(T, H, W)
    send = [wl.random_bits((part.tokens(r), P, H, D), 100 + r, DEV) for r in range(W)]
    recv = rr.alloc_head_side(T, P, H, D, W, DEV)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        rr.seq_to_head(send, recv, stream=s)
    s.synchronize()
    want = oracle_lib.seq_to_head([gu.bits(x) for x in send], T, P, H, D, W)
    for j in range(W):
        assert np.array_equal(gu.bits(recv[j]), want[j])


def test_chunked_plan_actually_ran():
    """The chunked plan reports one launch per plane; a window 16 bytes short
    of a plane splits every plane into two token chunks; an unchunked control
    reports one launch and fails the chunked assertion; a window that cannot
    hold one token of every rank is refused."""
    T, P, H, D, W = 1000, 4, 56, 128, 4
    full, send, part = _seq_inputs(T, P, H, D, W, seed=3)
    plane = max(part.tokens(0) * H * D * 2, T * part.heads(0) * D * 2)
    recv = rr.alloc_head_side(T, P, H, D, W, DEV)
    info = rr.seq_to_head(send, recv, window_bytes=plane)
    assert info["chunks"] == P and info["launches"] == P and info["planes_per_launch"] == 1
    info = rr.seq_to_head(send, recv, window_bytes=plane - 16)
    assert info["chunks"] == 2 * P and info["launches"] == 2 * P and info["planes_per_launch"] == 1
    assert rr.relayout_chunk_plan(T, P, H, D, W, plane - 16) == (125, 2 * P)
    control = rr.seq_to_head(send, recv, window_bytes=0)
    assert control["chunks"] == 1 and control["launches"] == 1
    with pytest.raises(AssertionError):
        assert control["launches"] == P
    with pytest.raises(rr.H3Error) as e:
        rr.seq_to_head(send, recv, window_bytes=H * D * 2 - 16)
    assert e.value.status == 4  # H3_ERR_WINDOW


# Planes larger than the window are split into token chunks (FastVideo PR
# #1807, "Problem and behavior": transfers bounded by the window): half a
# plane, and one token of every rank per launch; ragged tokens and heads,
# a head rank receiving more than a token row (W x H_max > H), one token per
# rank, narrow rows.
SUB_PLANE = [
    (1000, 3, 56, 128, 4),
    (1000, 3, 56, 128, 6),
    (777, 4, 56, 128, 8),
    (301, 2, 16, 64, 5),
    (130, 2, 7, 64, 3),
    (19, 3, 56, 128, 9),
]


@pytest.mark.parametrize("T,P,H,D,W", SUB_PLANE)
@pytest.mark.parametrize("kind", ["sub", "min"])
@pytest.mark.parametrize("variant", [0, rr.H3_VARIANT_BULK])
def test_sub_plane_chunks_match_oracle(oracle_lib, T, P, H, D, W, kind, variant):
    full, send, part = _seq_inputs(T, P, H, D, W, seed=T * 13 + W + len(kind))
    window = gu.chunk_window(kind, T, H, D, W)
    L, chunks = rr.relayout_chunk_plan(T, P, H, D, W, window)
    assert chunks > P  # every plane is split
    recv = rr.alloc_head_side(T, P, H, D, W, DEV)
    rr.bulk_wait_timeouts(reset=True)
    info = rr.seq_to_head(send, recv, window_bytes=window, variant=variant)
    assert info["chunks"] == chunks and info["launches"] == chunks
    want = oracle_lib.seq_to_head([gu.bits(s) for s in send], T, P, H, D, W)
    for j in range(W):
        assert np.array_equal(gu.bits(recv[j]), want[j]), f"seq->head rank {j}"
    back_full, back = rr.alloc_seq_side(T, P, H, D, W, DEV)
    info = rr.head_to_seq(recv, back, window_bytes=window, variant=variant)
    assert info["chunks"] == chunks and info["launches"] == chunks
    want_back = oracle_lib.head_to_seq(want, T, P, H, D, W)
    for r in range(W):
        assert np.array_equal(gu.bits(back[r]), want_back[r]), f"head->seq rank {r}"
    assert gu.same_bits(back_full, full)
    assert rr.bulk_wait_timeouts() == 0


@pytest.mark.parametrize("T,P,H,D,W", SUB_PLANE)
@pytest.mark.parametrize("kind", ["plane", "half", "min"])
@pytest.mark.parametrize("variant", [0, rr.H3_VARIANT_BULK])
def test_token_range_chunks_match_oracle(oracle_lib, T, P, H, D, W, kind, variant):
    """H3_LAUNCH_CHUNK_TOKENS: the window cut into token ranges of every
    plane; launches, chunks and planes per launch as the plan says, results
    equal to the oracle's in both directions."""
    full, send, part = _seq_inputs(T, P, H, D, W, seed=T * 17 + W + len(kind))
    window = gu.range_window(kind, T, P, H, D, W)
    L, chunks = rr.relayout_chunk_plan(T, P, H, D, W, window, token_chunks=True)
    recv = rr.alloc_head_side(T, P, H, D, W, DEV)
    rr.bulk_wait_timeouts(reset=True)
    info = rr.seq_to_head(send, recv, window_bytes=window, variant=variant, token_chunks=True)
    assert info["chunks"] == chunks and info["launches"] == chunks and info["planes_per_launch"] == P
    want = oracle_lib.seq_to_head([gu.bits(s) for s in send], T, P, H, D, W)
    for j in range(W):
        assert np.array_equal(gu.bits(recv[j]), want[j]), f"seq->head rank {j}"
    back_full, back = rr.alloc_seq_side(T, P, H, D, W, DEV)
    info = rr.head_to_seq(recv, back, window_bytes=window, variant=variant, token_chunks=True)
    assert info["chunks"] == chunks and info["launches"] == chunks and info["planes_per_launch"] == P
    want_back = oracle_lib.head_to_seq(want, T, P, H, D, W)
    for r in range(W):
        assert np.array_equal(gu.bits(back[r]), want_back[r]), f"head->seq rank {r}"
    assert gu.same_bits(back_full, full)
    assert rr.bulk_wait_timeouts() == 0


def test_token_range_chunks_guard_bands():
    """One-token ranges of every plane write nothing outside the outputs."""
    T, P, H, D, W = 257, 3, 56, 128, 6
    full, send, part = _seq_inputs(T, P, H, D, W, seed=43)
    window = gu.range_window("min", T, P, H, D, W)
    bufs, recv = [], []
    for j in range(W):
        b, r = gu.guarded((T, P, part.heads(j), D), DEV)
        bufs.append(b)
        recv.append(r)
    info = rr.seq_to_head(send, recv, window_bytes=window, token_chunks=True)
    assert info["launches"] == -(-T // W)
    assert all(gu.guards_intact(b) for b in bufs)
    back_bufs, back = [], []
    for r in range(W):
        b, o = gu.guarded((part.tokens(r), P, H, D), DEV)
        back_bufs.append(b)
        back.append(o)
    rr.head_to_seq(recv, back, window_bytes=window, token_chunks=True)
    assert all(gu.guards_intact(b) for b in back_bufs)
    for r in range(W):
        ts, te = int(part.token_starts[r]), int(part.token_starts[r + 1])
        assert gu.same_bits(back[r], full[ts:te])


def test_sub_plane_chunks_guard_bands():
    """One-token chunks write nothing outside the outputs."""
    T, P, H, D, W = 257, 3, 56, 128, 6
    full, send, part = _seq_inputs(T, P, H, D, W, seed=41)
    window = gu.chunk_window("min", T, H, D, W)
    bufs, recv = [], []
    for j in range(W):
        b, o = gu.guarded((T, P, part.heads(j), D), DEV)
        bufs.append(b)
        recv.append(o)
    rr.seq_to_head(send, recv, window_bytes=window)
    assert all(gu.guards_intact(b) for b in bufs)
    sbufs, back = [], []
    for r in range(W):
        b, o = gu.guarded((part.tokens(r), P, H, D), DEV)
        sbufs.append(b)
        back.append(o)
    rr.head_to_seq(recv, back, window_bytes=window)
    assert all(gu.guards_intact(b) for b in sbufs)
    assert gu.same_bits(torch.cat(back), full)


def test_overlapping_output_rejected_on_device():
    """An output over an input is refused before launch (all bytes in bounds)."""
    T, P, H, D, W = 64, 3, 56, 128, 2
    full, send, part = _seq_inputs(T, P, H, D, W, seed=4)
    recv = rr.alloc_head_side(T, P, H, D, W, DEV)
    alias = full.view(-1)[: recv[1].numel()].view(recv[1].shape)
    with pytest.raises(rr.H3Error) as e:
        rr.seq_to_head(send, [recv[0], alias])
    assert e.value.status == 1


def test_stress_alternating(oracle_lib):
    """100 rounds alternating direction and world size on one stream."""
    T, P, H, D = 999, 3, 56, 128
    x = wl.random_bits((T, P, H, D), 77, DEV)
    cur = x.clone()
    worlds = [2, 4, 6, 8, 3, 7, 1, 5]
    for it in range(100):
        W = worlds[it % len(worlds)]
        part = rr.partition(T, H, W)
        recv = rr.alloc_head_side(T, P, H, D, W, DEV)
        rr.seq_to_head(rr.split_rows(cur, part.token_starts), recv,
                       window_bytes=(0 if it % 3 else T * part.heads(0) * D * 2 + part.tokens(0) * H * D * 2))
        nxt = torch.empty_like(cur)
        rr.head_to_seq(recv, rr.split_rows(nxt, part.token_starts))
        cur = nxt
    torch.cuda.synchronize()
    assert gu.same_bits(cur, x)


# ---------------------------------------------------------------------------
# full-size workloads: sampled oracle elements + properties at any size
# ---------------------------------------------------------------------------

def _full_size_round_trip(o, w, planes=None, window=0, seed_offset=0, token_chunks=False):
    P = w.P if planes is None else planes
    full = wl.packed_operand(w, planes=P, device=DEV, seed_offset=seed_offset)
    bounds = wl.segment_bounds(w.T, w.n_segs, w.seed, w.seg_lengths)
    part = rr.partition(w.T, w.H, w.W, bounds)
    send = rr.split_rows(full, part.token_starts)
    recv = rr.alloc_head_side(w.T, P, w.H, w.D, w.W, DEV)
    info = rr.seq_to_head(send, recv, window_bytes=window, token_chunks=token_chunks)
    # torch slicing as a third opinion on every element
    for j in range(w.W):
        hs, he = int(part.head_starts[j]), int(part.head_starts[j + 1])
        assert gu.same_bits(recv[j], full[:, :, hs:he, :]), f"rank {j} differs from slicing"
    gu.sampled_check_seq_to_head(o, send, recv, w.T, P, w.H, w.D, w.W, seed=w.seed)
    back_full, back = rr.alloc_seq_side(w.T, P, w.H, w.D, w.W, DEV)
    info_back = rr.head_to_seq(recv, back, window_bytes=window, token_chunks=token_chunks)
    gu.sampled_check_head_to_seq(o, recv, back, w.T, P, w.H, w.D, w.W, seed=w.seed + 1)
    assert gu.same_bits(back_full, full)
    return info, info_back


def test_full_qkv_32k_w6(oracle_lib):
    w = wl.QKV_32K_W6
    info, _ = _full_size_round_trip(oracle_lib, w)
    assert info["launches"] == 1


def test_full_qkvg_128k_w4(oracle_lib):
    w = wl.QKVG_128K_W4
    _full_size_round_trip(oracle_lib, w)
    torch.cuda.empty_cache()


def test_full_attention_output_128k_w4(oracle_lib):
    """head->seq on the attention output [131072, 56, 128] (one plane)."""
    w = wl.QKVG_128K_W4
    part = rr.partition(w.T, w.H, w.W)
    heads = [wl.normal_bf16((w.T, 1, part.heads(j), w.D), w.seed + 10 + j, 1.0, DEV)
             for j in range(w.W)]
    out_full, out = rr.alloc_seq_side(w.T, 1, w.H, w.D, w.W, DEV)
    rr.head_to_seq(heads, out)
    gu.sampled_check_head_to_seq(oracle_lib, heads, out, w.T, 1, w.H, w.D, w.W, seed=5)
    assert gu.same_bits(out_full, torch.cat(heads, dim=2))
    torch.cuda.empty_cache()


def test_full_qkvg_250k_w4_chunked(oracle_lib):
    w = wl.QKVG_250K_W4_CHUNKED
    info, info_back = _full_size_round_trip(oracle_lib, w, window=w.window_bytes)
    for i in (info, info_back):
        assert i["chunks"] == 4 and i["launches"] == 4 and i["planes_per_launch"] == 1
    torch.cuda.empty_cache()


def test_full_qkvg_250k_w4_token_ranges(oracle_lib):
    """The long-sequence operand under the pages' window cut into token
    ranges of all four planes: 15,625 tokens of every rank per launch
    (896,000,000 bytes each way per rank, as one plane of one rank), 4
    launches per direction; every element against torch slicing, sampled
    elements against the oracle, the round trip exact."""
    w = wl.QKVG_250K_W4_CHUNKED
    assert rr.relayout_chunk_plan(w.T, w.P, w.H, w.D, w.W, w.window_bytes, token_chunks=True) == (15625, 4)
    info, info_back = _full_size_round_trip(oracle_lib, w, window=w.window_bytes, token_chunks=True)
    for i in (info, info_back):
        assert i["chunks"] == 4 and i["launches"] == 4 and i["planes_per_launch"] == 4
    torch.cuda.empty_cache()


def test_full_qkvg_250k_w4_bulk_kernels_and_both_cuts():
    """At the long-sequence size, the TMA bulk kernels give the vector
    kernels' bytes under both cuts of the pages' window (one plane per launch
    and token ranges of every plane), in both directions; the vector result
    is itself checked against the oracle in the tests above."""
    w = wl.QKVG_250K_W4_CHUNKED
    full = wl.packed_operand(w, device=DEV)
    part = rr.partition(w.T, w.H, w.W)
    send = rr.split_rows(full, part.token_starts)
    ref = rr.alloc_head_side(w.T, w.P, w.H, w.D, w.W, DEV)
    rr.seq_to_head(send, ref, window_bytes=w.window_bytes)
    got = rr.alloc_head_side(w.T, w.P, w.H, w.D, w.W, DEV)
    back_full, back = rr.alloc_seq_side(w.T, w.P, w.H, w.D, w.W, DEV)
    rr.bulk_wait_timeouts(reset=True)
    for tok in (False, True):
        for h in got:
            h.zero_()
        info = rr.seq_to_head(send, got, window_bytes=w.window_bytes, variant=rr.H3_VARIANT_BULK,
                              token_chunks=tok)
        assert info["variant"] == rr.H3_VARIANT_BULK and info["launches"] == 4
        for j in range(w.W):
            assert gu.same_bits(got[j], ref[j]), (tok, j)
        back_full.zero_()
        rr.head_to_seq(ref, back, window_bytes=w.window_bytes, variant=rr.H3_VARIANT_BULK,
                       token_chunks=tok)
        assert gu.same_bits(back_full, full), tok
    assert rr.bulk_wait_timeouts() == 0
    del full, send, ref, got, back_full, back
    torch.cuda.empty_cache()


def test_full_qkvg_250k_w2_sub_plane(oracle_lib):
    """The long-sequence operand over 2 ranks: one plane of one rank is
    1,792,000,000 bytes, twice the 896,000,000-byte window, so every plane
    moves in two token chunks."""
    w = wl.QKVG_250K_W2_CHUNKED
    assert rr.relayout_chunk_plan(w.T, w.P, w.H, w.D, w.W, w.window_bytes) == (62500, 8)
    info, info_back = _full_size_round_trip(oracle_lib, w, window=w.window_bytes)
    for i in (info, info_back):
        assert i["chunks"] == 8 and i["launches"] == 8 and i["planes_per_launch"] == 1
    torch.cuda.empty_cache()


def test_prepared_calls_and_inverse(oracle_lib):
    """Prepared calls equal the one-shot calls; the inverse of a prepared
    seq->head is the matching head->seq (the backward reusing the forward's
    plan); refilling the buffers in place between calls is picked up."""
    T, P, H, D, W = 1000, 3, 56, 128, 6
    full, send, part = _seq_inputs(T, P, H, D, W, seed=21)
    heads = rr.alloc_head_side(T, P, H, D, W, DEV)
    fwd = rr.prepare_seq_to_head(send, heads, layout=0)
    back_full, back = rr.alloc_seq_side(T, P, H, D, W, DEV)
    bwd = fwd.inverse(heads, back)
    for round_ in range(3):
        full.copy_(wl.random_bits((T, P, H, D), 30 + round_, DEV))
        info = fwd()
        assert info.launches == 1
        bwd()
        torch.cuda.synchronize()
        want = oracle_lib.seq_to_head([gu.bits(s) for s in send], T, P, H, D, W)
        for j in range(W):
            assert np.array_equal(gu.bits(heads[j]), want[j])
        assert gu.same_bits(back_full, full)
    # prepared token-range chunks, and their inverse, keep the option
    window = gu.range_window("half", T, P, H, D, W)
    chunks = rr.relayout_chunk_plan(T, P, H, D, W, window, token_chunks=True)[1]
    fwd = rr.prepare_seq_to_head(send, heads, window_bytes=window, token_chunks=True)
    bwd = fwd.inverse(heads, back)
    assert bwd.token_chunks
    full.copy_(wl.random_bits((T, P, H, D), 40, DEV))
    assert fwd().launches == chunks and bwd().launches == chunks
    torch.cuda.synchronize()
    want = oracle_lib.seq_to_head([gu.bits(s) for s in send], T, P, H, D, W)
    for j in range(W):
        assert np.array_equal(gu.bits(heads[j]), want[j])
    assert gu.same_bits(back_full, full)
    with pytest.raises(ValueError):
        rr.prepare_seq_to_head(send, heads[:-1])
