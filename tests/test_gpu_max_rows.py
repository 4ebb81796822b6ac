"""The largest sizes the calls accept: T * P = 2^31 - 1 rows, the int32 row
limit every entry point checks (2^31 rows are refused before any launch,
see tests/test_abi_cpu.py).  Rows of 16 bytes keep each buffer at 34.4 GB;
the last row's byte offset is above 2^35, so any 32-bit index or offset
anywhere in a kernel would show.

Relayouts run at W = 1 (the only world that fits: every rank needs a head,
and a head row is at least 16 bytes), where the oracle's result is the
identity; the whole output is compared with the input on the device and
sampled elements through the oracle's locate functions.  Reduce-scatter and
all-gather run at W = 2 (a ragged split: 2^30 and 2^30 - 1 rows): sampled
rows through the oracle, including both ranks' first and last rows, and
every element against torch's binary32 adds in the same order."""
import numpy as np
import pytest
import torch

import ragged_reduce_b200 as rr
import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

DEV = "cuda"
MAX_ROWS = 2**31 - 1
CHUNK = 1 << 28  # elements compared per step on the device


@pytest.fixture(autouse=True)
def _release_memory():
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()  # hand the ~100 GB back before the next test


def _need(nbytes):
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    free = torch.cuda.mem_get_info()[0]
    if free < nbytes + (8 << 30):
        pytest.skip(f"needs {nbytes / 2**30:.0f} GiB free on the device, {free / 2**30:.0f} free")


def _same_in_chunks(a, b):
    x = a.view(-1).view(torch.int16)
    y = b.view(-1).view(torch.int16)
    assert x.numel() == y.numel()
    for lo in range(0, x.numel(), CHUNK):
        hi = min(x.numel(), lo + CHUNK)
        if not torch.equal(x[lo:hi], y[lo:hi]):
            return False
    return True


def _sample_elems(n, seed):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([rng.integers(0, n, 4096), np.arange(16), n - 1 - np.arange(16)]))


def test_relayouts_at_the_row_limit(oracle_lib):
    T, P, H, D, W = MAX_ROWS, 1, 1, 8, 1
    nbytes = T * P * H * D * 2
    _need(2 * nbytes)
    send = wl.normal_bf16((T, P, H, D), 2031, 1.0, DEV)
    heads = [torch.empty((T, P, H, D), dtype=torch.bfloat16, device=DEV)]
    info = rr.seq_to_head([send], heads)
    assert info["launches"] == 1
    torch.cuda.synchronize()
    assert _same_in_chunks(heads[0], send)
    elems = _sample_elems(T * P * H * D, 1)
    src_rank, src_elem = oracle_lib.seq_to_head_locate(T, P, H, D, W, 0, elems)
    assert np.all(src_rank == 0)
    flat_in = send.view(-1).view(torch.int16)
    flat_out = heads[0].view(-1).view(torch.int16)
    got = flat_out.index_select(0, torch.from_numpy(elems).to(DEV)).cpu().numpy()
    src_t = torch.from_numpy(np.asarray(src_elem, dtype=np.int64)).to(DEV)
    want = flat_in.index_select(0, src_t).cpu().numpy()
    assert np.array_equal(got, want)

    # head->seq back into the (overwritten) sequence-side buffer
    keep = flat_in.index_select(0, torch.from_numpy(elems).to(DEV)).cpu().numpy()
    send.view(torch.int16).fill_(0x7fc1)
    rr.head_to_seq(heads, [send])
    torch.cuda.synchronize()
    assert _same_in_chunks(send, heads[0])
    assert np.array_equal(flat_in.index_select(0, torch.from_numpy(elems).to(DEV)).cpu().numpy(), keep)
    del send, heads, flat_in, flat_out


def test_token_chunked_relayouts_at_the_row_limit(oracle_lib):
    """A window of a third of the plane: the plane of 2^31 - 1 rows moves in
    three token chunks, the last starting above row 2^30 (chunk offsets and
    rows stay in the kernels' 32-bit range; byte offsets above 2^35)."""
    T, P, H, D, W = MAX_ROWS, 1, 1, 8, 1
    nbytes = T * P * H * D * 2
    _need(2 * nbytes)
    window = nbytes // 3 + 16
    L, chunks = rr.relayout_chunk_plan(T, P, H, D, W, window)
    assert chunks == 3 and 2 * L < T <= 3 * L
    send = wl.normal_bf16((T, P, H, D), 2034, 1.0, DEV)
    heads = [torch.empty((T, P, H, D), dtype=torch.bfloat16, device=DEV)]
    info = rr.seq_to_head([send], heads, window_bytes=window)
    assert info["launches"] == 3 and info["chunks"] == 3
    torch.cuda.synchronize()
    assert _same_in_chunks(heads[0], send)
    elems = _sample_elems(T * P * H * D, 3)
    flat_in = send.view(-1).view(torch.int16)
    keep = flat_in.index_select(0, torch.from_numpy(elems).to(DEV)).cpu().numpy()
    src_rank, src_elem = oracle_lib.head_to_seq_locate(T, P, H, D, W, 0, elems)
    assert np.all(src_rank == 0) and np.array_equal(np.asarray(src_elem), elems)
    send.view(torch.int16).fill_(0x7fc1)
    info = rr.head_to_seq(heads, [send], window_bytes=window)
    assert info["launches"] == 3
    torch.cuda.synchronize()
    assert _same_in_chunks(send, heads[0])
    assert np.array_equal(flat_in.index_select(0, torch.from_numpy(elems).to(DEV)).cpu().numpy(), keep)
    del send, heads, flat_in


def test_reduce_scatter_and_all_gather_at_the_row_limit(oracle_lib):
    T, C, W = MAX_ROWS, 8, 2
    row_bytes = C * 2
    _need((W + 1) * T * row_bytes)
    partials = wl.normal_bf16((W, T, C), 2032, 0.5, DEV)
    bias = wl.normal_bf16((C,), 2033, 0.1, DEV)
    out_full, out = rr.alloc_reduce_outputs(T, C, W, DEV)
    part = rr.partition(T, W, W)
    assert [o.shape[0] for o in out] == [2**30, 2**30 - 1]
    info = rr.ragged_reduce_scatter(partials, bias, out)
    assert info["launches"] == 1
    torch.cuda.synchronize()

    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([rng.integers(0, T, 2048), part.token_starts[:-1],
                                     part.token_starts[1:] - 1]))
    rows_t = torch.from_numpy(rows).to(DEV)
    want = oracle_lib.reduce_rows([gu.bits(partials[k].index_select(0, rows_t)) for k in range(W)],
                                  gu.bits(bias))
    assert np.array_equal(gu.bits(out_full.index_select(0, rows_t)), want)
    for r in range(W):
        assert out[r].data_ptr() == out_full[int(part.token_starts[r])].data_ptr()
    step = CHUNK // C
    bias_f = bias.float()
    for lo in range(0, T, step):
        hi = min(T, lo + step)
        acc = partials[0, lo:hi].float()
        acc += partials[1, lo:hi].float()
        acc += bias_f
        assert gu.same_bits(out_full[lo:hi], acc.to(torch.bfloat16)), lo
        del acc
    del partials

    # all-gather of the reduced rows to both ranks
    _need(W * T * row_bytes)
    gathered = [torch.empty((T, C), dtype=torch.bfloat16, device=DEV) for _ in range(W)]
    info = rr.ragged_all_gather(out, gathered)
    assert info["launches"] == 1
    torch.cuda.synchronize()
    for g in gathered:
        assert _same_in_chunks(g, out_full)
