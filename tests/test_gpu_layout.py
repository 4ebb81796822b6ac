"""GPU parity of the relayouts with plane-major buffers against the oracle."""
import numpy as np
import pytest
import torch

import ragged_reduce_b200 as rr
import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

DEV = "cuda"
SPM = rr.H3_LAYOUT_SEQ_PLANE_MAJOR
HPM = rr.H3_LAYOUT_HEAD_PLANE_MAJOR


def _seq_buffers(T, P, H, D, W, seq_pm, seed):
    part = rr.partition(T, H, W)
    if seq_pm:
        return [wl.random_bits((P, part.tokens(r), H, D), seed + r, DEV) for r in range(W)], part
    full = wl.random_bits((T, P, H, D), seed, DEV)
    return rr.split_rows(full, part.token_starts), part


def _head_buffers(T, P, H, D, W, head_pm, part):
    shape = (lambda j: (P, T, part.heads(j), D)) if head_pm else (lambda j: (T, P, part.heads(j), D))
    return [torch.empty(shape(j), dtype=torch.bfloat16, device=DEV) for j in range(W)]


@pytest.mark.parametrize("T,P,H,D,W", [(1000, 3, 56, 128, 6), (777, 4, 56, 128, 8),
                                       (130, 2, 7, 64, 3), (50, 3, 5, 8, 5), (20, 2, 300, 128, 7),
                                       (33, 3, 56, 256, 4), (64, 3, 56, 128, 1)])
@pytest.mark.parametrize("layout", [0, SPM, HPM, SPM | HPM])
@pytest.mark.parametrize("chunked", [None, "plane", "sub", "ranges"])
def test_layout_matches_oracle(oracle_lib, T, P, H, D, W, layout, chunked):
    spm, hpm = bool(layout & SPM), bool(layout & HPM)
    send, part = _seq_buffers(T, P, H, D, W, spm, seed=T + W + layout)
    heads = _head_buffers(T, P, H, D, W, hpm, part)
    ranges = chunked == "ranges"  # token ranges of every plane (H3_LAUNCH_CHUNK_TOKENS)
    window = gu.range_window("half", T, P, H, D, W) if ranges else gu.chunk_window(chunked, T, H, D, W)
    info = rr.seq_to_head_layout(send, heads, layout, window_bytes=window, token_chunks=ranges)
    assert info["launches"] == rr.relayout_chunk_plan(T, P, H, D, W, window, token_chunks=ranges)[1]
    want = oracle_lib.relayout_layout([gu.bits(s) for s in send], T, P, H, D, W, True, spm, hpm)
    for j in range(W):
        assert np.array_equal(gu.bits(heads[j]), want[j]), f"seq->head rank {j}"
    back = [torch.empty_like(s) for s in send]
    rr.head_to_seq_layout(heads, back, layout, window_bytes=window, token_chunks=ranges)
    for r in range(W):
        assert gu.same_bits(back[r], send[r]), f"round trip rank {r}"


def test_head_plane_major_gives_contiguous_qkv_full_size():
    """128k-token QKVG over 4 ranks: plane p of head rank j is x[:, p, hs_j:he_j]."""
    w = wl.QKVG_128K_W4
    x = wl.packed_operand(w, device=DEV)
    part = rr.partition(w.T, w.H, w.W)
    send = rr.split_rows(x, part.token_starts)
    heads = [torch.empty((w.P, w.T, part.heads(j), w.D), dtype=torch.bfloat16, device=DEV)
             for j in range(w.W)]
    rr.seq_to_head_layout(send, heads, HPM)
    for j in range(w.W):
        hs, he = int(part.head_starts[j]), int(part.head_starts[j + 1])
        for p in range(w.P):
            q = heads[j][p]
            assert q.is_contiguous()
            assert gu.same_bits(q, x[:, p, hs:he, :])
    del heads
    torch.cuda.empty_cache()


def test_layout_rejects_bulk_and_unknown_bits():
    T, P, H, D, W = 64, 3, 56, 128, 2
    send, part = _seq_buffers(T, P, H, D, W, False, 1)
    heads = _head_buffers(T, P, H, D, W, True, part)
    with pytest.raises(rr.H3Error) as e:
        rr.seq_to_head_layout(send, heads, HPM, variant=rr.H3_VARIANT_BULK)
    assert e.value.status == 5
