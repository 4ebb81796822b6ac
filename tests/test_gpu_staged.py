"""GPU parity of the staged (window) relayouts against the CPU oracle.

The staged calls pack each chunk (one plane, a run of tokens) into a window
buffer and unpack it; the results must equal the oracle bit for bit for any
window size from one token row up, and the kernels must write nothing
outside the window and the outputs."""
import numpy as np
import pytest
import torch

import ragged_reduce_b200 as rr
import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

DEV = "cuda"

# T, P, H, D, W, window bytes: one token row, a few rows with a ragged last
# chunk, exactly one plane, more than the whole operand, narrow heads.
CASES = [
    (1024, 3, 56, 128, 2, 100 * 14336),
    (1000, 3, 56, 128, 6, 7 * 14336 + 100),
    (777, 4, 56, 128, 8, 14336),
    (130, 2, 7, 64, 3, 5 * 896),
    (50, 3, 5, 8, 5, 80 * 7),
    (9, 3, 56, 128, 9, 4 * 14336),
    (64, 3, 56, 128, 56, 64 * 14336),
    (300, 1, 24, 128, 7, 33 * 6144),
    (200, 3, 56, 128, 4, 10_000_000),
]


def _window(nbytes):
    """A window with canary bands on both sides (int16 elements)."""
    n = (nbytes + 15) // 16 * 8
    buf = torch.full((n + 2 * gu.GUARD_ELEMS,), gu.CANARY, dtype=torch.int16, device=DEV)
    return buf, buf[gu.GUARD_ELEMS:gu.GUARD_ELEMS + n]


@pytest.mark.parametrize("T,P,H,D,W,wbytes", CASES)
def test_staged_matches_oracle(oracle_lib, T, P, H, D, W, wbytes):
    full = wl.random_bits((T, P, H, D), T + W, DEV)
    part = rr.partition(T, H, W)
    send = rr.split_rows(full, part.token_starts)
    heads = rr.alloc_head_side(T, P, H, D, W, DEV)
    buf, win = _window(wbytes)
    n_tok, chunks = rr.staged_plan(T, P, H, D, win.numel() * 2)
    info = rr.seq_to_head_staged(send, heads, win)
    assert info["chunks"] == chunks and info["launches"] == 2 * chunks
    assert info["variant"] == rr.H3_VARIANT_STAGED
    want = oracle_lib.seq_to_head([gu.bits(s) for s in send], T, P, H, D, W)
    for j in range(W):
        assert np.array_equal(gu.bits(heads[j]), want[j]), f"seq->head rank {j}"
    back_full, back = rr.alloc_seq_side(T, P, H, D, W, DEV)
    info = rr.head_to_seq_staged(heads, back, win)
    assert info["chunks"] == chunks
    assert gu.same_bits(back_full, full)
    assert gu.guards_intact(buf)


def test_staged_equals_direct_on_full_qkv_32k():
    w = wl.QKV_32K_W6
    x = wl.packed_operand(w, device=DEV)
    part = rr.partition(w.T, w.H, w.W)
    send = rr.split_rows(x, part.token_starts)
    direct = rr.alloc_head_side(w.T, w.P, w.H, w.D, w.W, DEV)
    rr.seq_to_head(send, direct)
    staged = rr.alloc_head_side(w.T, w.P, w.H, w.D, w.W, DEV)
    win = torch.empty(64 << 20, dtype=torch.uint8, device=DEV)
    info = rr.seq_to_head_staged(send, staged, win)
    assert info["chunks"] == rr.staged_plan(w.T, w.P, w.H, w.D, 64 << 20)[1]
    for j in range(w.W):
        assert gu.same_bits(staged[j], direct[j])
    back_full, back = rr.alloc_seq_side(w.T, w.P, w.H, w.D, w.W, DEV)
    rr.head_to_seq_staged(staged, back, win)
    assert gu.same_bits(back_full, x)


def test_staged_full_250k_qkvg_with_the_pages_window():
    """The pages' configuration: QKVG [250000, 4, 56, 128] over 4 ranks
    through an 896,000,000-byte window: staged equals direct in both
    directions.  The window holds 62,500 full token rows, so each plane
    takes 4 chunks (16 per direction)."""
    w = wl.QKVG_250K_W4_CHUNKED
    x = wl.packed_operand(w, device=DEV)
    part = rr.partition(w.T, w.H, w.W)
    send = rr.split_rows(x, part.token_starts)
    win = torch.empty(w.window_bytes, dtype=torch.uint8, device=DEV)
    staged = rr.alloc_head_side(w.T, w.P, w.H, w.D, w.W, DEV)
    info = rr.seq_to_head_staged(send, staged, win)
    assert info["chunks"] == 16 and info["launches"] == 32
    assert rr.staged_plan(w.T, w.P, w.H, w.D, w.window_bytes) == (62500, 16)
    direct = rr.alloc_head_side(w.T, w.P, w.H, w.D, w.W, DEV)
    rr.seq_to_head(send, direct, window_bytes=w.window_bytes)
    for j in range(w.W):
        assert gu.same_bits(staged[j], direct[j]), j
    del direct
    torch.cuda.empty_cache()
    back_full, back = rr.alloc_seq_side(w.T, w.P, w.H, w.D, w.W, DEV)
    rr.head_to_seq_staged(staged, back, win)
    assert gu.same_bits(back_full, x)


def test_staged_rejects_small_or_overlapping_window():
    T, P, H, D, W = 100, 3, 56, 128, 4
    full = wl.random_bits((T, P, H, D), 3, DEV)
    part = rr.partition(T, H, W)
    send = rr.split_rows(full, part.token_starts)
    heads = rr.alloc_head_side(T, P, H, D, W, DEV)
    with pytest.raises(rr.H3Error) as e:
        rr.seq_to_head_staged(send, heads, torch.empty(14336 - 16, dtype=torch.uint8, device=DEV))
    assert e.value.status == 4  # H3_ERR_WINDOW
    with pytest.raises(rr.H3Error) as e:
        rr.seq_to_head_staged(send, heads, full.view(-1)[:7168])  # window inside an input
    assert e.value.status == 1
