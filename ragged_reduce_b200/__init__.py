"""B200-native (sm_100a) H3 Ulysses relayouts and tensor-mode ragged reduce-scatter.

Python binding of ``include/h3rr.h``: argument marshalling only.  Every byte
the calls produce is computed by the library's own CUDA kernels; there is no
CPU or PyTorch fallback, and importing this package fails if ``libh3rr.so``
is missing.

Terms ("Distributed H3 Execution", sections intro and "Partition Contract"):
W virtual ranks; T packed tokens split by quotient/remainder into token ranges
[ts_r, te_r); H heads (56 for H3) split the same way into head ranges
[hs_j, he_j); P planes of a packed operand (3 for QKV, 4 for QKVG, 1 for the
attention output); D = 128 values per head.

* ``partition``                - host: token/head ranges and clipped, rebased segments
* ``seq_to_head``              - sequence side [T_r, P, H, D] -> head side [T, P, H_j, D]
* ``head_to_seq``              - head side -> sequence side
* ``ragged_reduce_scatter``    - W partials [T, C] -> rank rows [T_r, C], bias once
"""
from __future__ import annotations

import contextlib
import ctypes as C
import functools
from dataclasses import dataclass

import numpy as np
import torch

from . import _abi
from ._abi import (ExecInfo, H3Error, LaunchConfig, H3_LAYOUT_HEAD_PLANE_MAJOR,
                   H3_LAYOUT_SEQ_PLANE_MAJOR, H3_VARIANT_BULK, H3_VARIANT_GATHER,
                   H3_VARIANT_REDUCE, H3_VARIANT_STAGED, H3_VARIANT_VECTOR, H3_LAUNCH_SERIAL,
                   H3_LAUNCH_CHUNK_TOKENS, MAX_WORLD)

__all__ = [
    "H3Error", "Partition", "partition", "seq_to_head", "head_to_seq",
    "ragged_reduce_scatter", "alloc_head_side", "alloc_seq_side", "split_rows",
    "H3_VARIANT_VECTOR", "H3_VARIANT_BULK", "H3_VARIANT_REDUCE", "MAX_WORLD", "library_path",
    "bulk_wait_timeouts", "alloc_reduce_outputs", "seq_to_head_staged", "head_to_seq_staged",
    "staged_plan", "relayout_chunk_plan", "relayout_launch_plan", "H3_VARIANT_STAGED",
    "ragged_all_gather", "H3_VARIANT_GATHER",
    "seq_to_head_layout", "head_to_seq_layout", "H3_LAYOUT_SEQ_PLANE_MAJOR",
    "H3_LAYOUT_HEAD_PLANE_MAJOR", "ragged_reduce_scatter_gated", "PreparedRelayout", "H3_LAUNCH_SERIAL",
    "H3_LAUNCH_CHUNK_TOKENS",
    "PreparedReduceScatter", "prepare_seq_to_head", "prepare_head_to_seq",
    "seq_to_head_rank", "head_to_seq_rank", "ragged_reduce_scatter_rank", "ragged_all_gather_rank",
    "ragged_reduce_scatter_gated_rank", "bounded_wait_selftest",
    "prepare_ragged_reduce_scatter",
]

library_path = _abi.LIB_PATH


@dataclass
class Partition:
    """Result of ``partition``: ranges per rank and each rank's rebased segments."""

    token_starts: np.ndarray          # int64 [W+1]
    head_starts: np.ndarray           # int32 [W+1]
    local_bounds: list                # per rank: int64 [pieces+1], 0 .. T_r
    seg_ids: list                     # per rank: int32 [pieces], global segment index

    @property
    def world(self) -> int:
        return len(self.token_starts) - 1

    def tokens(self, r: int) -> int:
        """Tokens rank r owns (te_r - ts_r)."""
        return int(self.token_starts[r + 1] - self.token_starts[r])

    def heads(self, j: int) -> int:
        """Heads rank j owns (he_j - hs_j)."""
        return int(self.head_starts[j + 1] - self.head_starts[j])


def partition(n_tokens: int, n_heads: int, world: int, seg_bounds=None) -> Partition:
    """Token and head ranges of every rank, and the packed segments clipped to
    each rank's token range and rebased to it (``h3_partition``)."""
    W = int(world)
    ts = np.zeros(max(W, 0) + 1, dtype=np.int64)
    hs = np.zeros(max(W, 0) + 1, dtype=np.int32)
    if seg_bounds is None:
        st = _abi.lib.h3_partition(int(n_tokens), int(n_heads), W, None, 0,
                                   ts.ctypes.data_as(_abi._i64p), hs.ctypes.data_as(_abi._i32p),
                                   None, None, None)
        _abi.check(st, "h3_partition")
        return Partition(ts, hs, [], [])
    b = np.ascontiguousarray(seg_bounds, dtype=np.int64)
    S = len(b) - 1
    if S < 1:
        raise ValueError("seg_bounds needs at least two boundaries")
    lb = np.zeros(S + 2 * W - 1, dtype=np.int64)
    ids = np.zeros(S + W - 1, dtype=np.int32)
    off = np.zeros(W + 1, dtype=np.int32)
    st = _abi.lib.h3_partition(int(n_tokens), int(n_heads), W, b.ctypes.data_as(_abi._i64p), S,
                               ts.ctypes.data_as(_abi._i64p), hs.ctypes.data_as(_abi._i32p),
                               lb.ctypes.data_as(_abi._i64p), ids.ctypes.data_as(_abi._i32p),
                               off.ctypes.data_as(_abi._i32p))
    _abi.check(st, "h3_partition")
    bounds = [lb[off[r] + r: off[r + 1] + r + 1].copy() for r in range(W)]
    seg = [ids[off[r]: off[r + 1]].copy() for r in range(W)]
    return Partition(ts, hs, bounds, seg)


# ---------------------------------------------------------------------------
# buffer helpers (allocation is the caller's; these use torch's allocator)
# ---------------------------------------------------------------------------

def split_rows(x: torch.Tensor, starts) -> list:
    """Views of x's leading dimension at the given rank starts."""
    return [x[int(starts[r]):int(starts[r + 1])] for r in range(len(starts) - 1)]


def alloc_head_side(T: int, P: int, H: int, D: int, W: int, device, dtype=torch.bfloat16):
    """One [T, P, H_j, D] buffer per head-side rank."""
    part = partition(T, H, W)
    return [torch.empty((T, P, part.heads(j), D), dtype=dtype, device=device) for j in range(W)]


def alloc_seq_side(T: int, P: int, H: int, D: int, W: int, device, dtype=torch.bfloat16):
    """One [T, P, H, D] tensor and its per-rank [T_r, P, H, D] views."""
    part = partition(T, H, W)
    full = torch.empty((T, P, H, D), dtype=dtype, device=device)
    return full, split_rows(full, part.token_starts)


# ---------------------------------------------------------------------------
# marshalling
# ---------------------------------------------------------------------------

def _as_list(x):
    if isinstance(x, torch.Tensor):
        return list(x.unbind(0))
    return list(x)


def _check_tensors(ts, what: str, itemsize: int = 2):
    index = None
    for t in ts:
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{what}: expected torch tensors")
        if not t.is_cuda:
            raise ValueError(f"{what}: tensors must be on a CUDA device (got {t.device})")
        if t.element_size() != itemsize:
            raise ValueError(f"{what}: expected {itemsize}-byte elements (got {t.dtype})")
        if not t.is_contiguous():
            raise ValueError(f"{what}: tensors must be contiguous")
        i = t.get_device()
        if index is None:
            index = i
        elif i != index:
            raise ValueError(f"{what}: all tensors must be on one device")
    return torch.device("cuda", index) if index is not None else None


def _device_guard(dev):
    """Make `dev` the current device for the call (no-op when it already is)."""
    if dev is None or dev.index is None or dev.index == torch.cuda.current_device():
        return contextlib.nullcontext()
    return torch.cuda.device(dev)


@functools.lru_cache(maxsize=1024)
def _rank_sizes(n_tokens: int, n_heads: int, world: int) -> tuple:
    """(tokens per rank, heads per rank) as ``h3_partition`` assigns them,
    cached per shape so that repeated calls pay one dictionary lookup.  Raises
    the library's error (for example an empty partition) like ``partition``."""
    p = partition(n_tokens, n_heads, world)
    return (tuple(int(v) for v in np.diff(p.token_starts)),
            tuple(int(v) for v in np.diff(p.head_starts)))


def _stream_handle(stream, device) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _flags(serial: bool = False, token_chunks: bool = False) -> int:
    return (H3_LAUNCH_SERIAL if serial else 0) | (H3_LAUNCH_CHUNK_TOKENS if token_chunks else 0)


def _config(variant: int, ctas_per_sm: int, serial: bool = False, token_chunks: bool = False):
    if not variant and not ctas_per_sm and not serial and not token_chunks:
        return None
    return C.byref(LaunchConfig(int(variant), int(ctas_per_sm), _flags(serial, token_chunks), 0))


def _relayout_shapes(seq_to_head_dir: bool, send, recv, layout: int = 0):
    """Check the per-rank shapes; return (T, P, H, D, W, device)."""
    W = len(send)
    if W < 1 or len(recv) != W:
        raise ValueError("send and recv need one tensor per rank (same count)")
    dev = _check_tensors(send + recv, "relayout")
    seq_side = send if seq_to_head_dir else recv
    head_side = recv if seq_to_head_dir else send
    if any(t.dim() != 4 for t in send + recv):
        raise ValueError("relayout buffers are 4-D: [tokens, planes, heads, head_dim]")
    seq_pm = bool(layout & _abi.H3_LAYOUT_SEQ_PLANE_MAJOR)
    head_pm = bool(layout & _abi.H3_LAYOUT_HEAD_PLANE_MAJOR)
    if seq_pm:
        P, _, H, D = seq_side[0].shape
        T = sum(int(t.shape[1]) for t in seq_side)
    else:
        _, P, H, D = seq_side[0].shape
        T = sum(int(t.shape[0]) for t in seq_side)
    tok, hds = _rank_sizes(T, int(H), W)  # raises the library's H3_ERR_EMPTY_PARTITION
    for r, t in enumerate(seq_side):
        want = (P, tok[r], H, D) if seq_pm else (tok[r], P, H, D)
        if tuple(t.shape) != want:
            raise ValueError(f"sequence-side rank {r}: shape {tuple(t.shape)}, expected {want}")
    for j, t in enumerate(head_side):
        want = (P, T, hds[j], D) if head_pm else (T, P, hds[j], D)
        if tuple(t.shape) != want:
            raise ValueError(f"head-side rank {j}: shape {tuple(t.shape)}, expected {want}")
    return T, int(P), int(H), int(D), W, dev


def _relayout_layout(seq_to_head_dir: bool, send, recv, layout, window_bytes, stream, variant,
                     ctas_per_sm, serial=False, token_chunks=False):
    send = _as_list(send)
    recv = _as_list(recv)
    T, P, H, D, W, dev = _relayout_shapes(seq_to_head_dir, send, recv, layout)
    info = ExecInfo()
    name = "h3_seq_to_head_layout" if seq_to_head_dir else "h3_head_to_seq_layout"
    cfg = _config(variant, ctas_per_sm, serial, token_chunks)
    with _device_guard(dev):
        st = getattr(_abi.lib, name)(
            _abi.pointer_array([t.data_ptr() for t in send]),
            _abi.pointer_array([t.data_ptr() for t in recv]),
            T, P, H, D, W, int(window_bytes), int(layout), C.c_void_p(_stream_handle(stream, dev)),
            cfg, C.byref(info))
    _abi.check(st, name)
    return info.as_dict()


def seq_to_head_layout(send, recv, layout: int, *, window_bytes: int = 0, stream=None,
                       variant: int = 0, ctas_per_sm: int = 0, serial: bool = False,
                       token_chunks: bool = False) -> dict:
    """seq->head with plane-major buffers (``layout``: bit set of
    H3_LAYOUT_SEQ_PLANE_MAJOR / H3_LAYOUT_HEAD_PLANE_MAJOR).  Plane-major
    sequence side: W tensors [P, T_r, H, D]; plane-major head side: W tensors
    [P, T, H_j, D] (out[j][0], [1], [2] are that rank's Q, K, V)."""
    return _relayout_layout(True, send, recv, layout, window_bytes, stream, variant, ctas_per_sm,
                            serial, token_chunks)


def head_to_seq_layout(send, recv, layout: int, *, window_bytes: int = 0, stream=None,
                       variant: int = 0, ctas_per_sm: int = 0, serial: bool = False,
                       token_chunks: bool = False) -> dict:
    """head->seq with plane-major buffers (see ``seq_to_head_layout``)."""
    return _relayout_layout(False, send, recv, layout, window_bytes, stream, variant, ctas_per_sm,
                            serial, token_chunks)


def _relayout_staged(seq_to_head_dir: bool, send, recv, window, stream):
    send = _as_list(send)
    recv = _as_list(recv)
    T, P, H, D, W, dev = _relayout_shapes(seq_to_head_dir, send, recv)
    _check_tensors([window], "window", itemsize=window.element_size())
    if window.device != dev:
        raise ValueError("window must be on the buffers' device")
    nbytes = window.numel() * window.element_size()
    info = ExecInfo()
    name = "h3_seq_to_head_staged" if seq_to_head_dir else "h3_head_to_seq_staged"
    with _device_guard(dev):
        st = getattr(_abi.lib, name)(
            _abi.pointer_array([t.data_ptr() for t in send]),
            _abi.pointer_array([t.data_ptr() for t in recv]),
            T, P, H, D, W, C.c_void_p(window.data_ptr()), int(nbytes),
            C.c_void_p(_stream_handle(stream, dev)), C.byref(info))
    _abi.check(st, name)
    return info.as_dict()


def seq_to_head_staged(send, recv, window: torch.Tensor, *, stream=None) -> dict:
    """seq->head staged through a window buffer (any contiguous CUDA tensor;
    its byte size is the window): chunks of one plane and as many tokens as
    fit, packed into the window and unpacked.  Same result as ``seq_to_head``."""
    return _relayout_staged(True, send, recv, window, stream)


def head_to_seq_staged(send, recv, window: torch.Tensor, *, stream=None) -> dict:
    """head->seq staged through a window buffer (see ``seq_to_head_staged``)."""
    return _relayout_staged(False, send, recv, window, stream)


def staged_plan(n_tokens: int, planes: int, n_heads: int, head_dim: int, window_bytes: int):
    """(tokens per chunk, chunks) of a staged call (``h3_staged_plan``, host only)."""
    n = C.c_int64(0)
    k = C.c_int64(0)
    st = _abi.lib.h3_staged_plan(int(n_tokens), int(planes), int(n_heads), int(head_dim),
                                 int(window_bytes), C.byref(n), C.byref(k))
    _abi.check(st, "h3_staged_plan")
    return int(n.value), int(k.value)


def relayout_chunk_plan(n_tokens: int, planes: int, n_heads: int, head_dim: int, world: int,
                        window_bytes: int, *, token_chunks: bool = False):
    """(tokens of each rank per launch, launches) of a chunked relayout
    (``h3_relayout_chunk_plan_ex``, host only): one batch plane per launch, a
    plane larger than the window split into equal token chunks; with
    token_chunks=True, equal token ranges of every plane instead."""
    n = C.c_int64(0)
    k = C.c_int64(0)
    st = _abi.lib.h3_relayout_chunk_plan_ex(int(n_tokens), int(planes), int(n_heads), int(head_dim),
                                            int(world), int(window_bytes), _flags(False, token_chunks),
                                            C.byref(n), C.byref(k), None)
    _abi.check(st, "h3_relayout_chunk_plan_ex")
    return int(n.value), int(k.value)


def relayout_launch_plan(n_tokens: int, planes: int, n_heads: int, head_dim: int, world: int,
                         window_bytes: int, *, token_chunks: bool = False) -> dict:
    """The launches a relayout call will make (``h3_relayout_chunk_plan_ex``,
    host only): {"tokens_per_launch": L (tokens of each rank, the last launch
    of a plane group may hold fewer), "launches": count, "planes_per_launch":
    1 one plane per launch or P}."""
    n = C.c_int64(0)
    k = C.c_int64(0)
    per = C.c_int32(0)
    st = _abi.lib.h3_relayout_chunk_plan_ex(int(n_tokens), int(planes), int(n_heads), int(head_dim),
                                            int(world), int(window_bytes), _flags(False, token_chunks),
                                            C.byref(n), C.byref(k), C.byref(per))
    _abi.check(st, "h3_relayout_chunk_plan_ex")
    return {"tokens_per_launch": int(n.value), "launches": int(k.value),
            "planes_per_launch": int(per.value)}


def _relayout(seq_to_head_dir: bool, send, recv, window_bytes, stream, variant, ctas_per_sm,
              serial=False, token_chunks=False):
    send = _as_list(send)
    recv = _as_list(recv)
    T, P, H, D, W, dev = _relayout_shapes(seq_to_head_dir, send, recv)
    info = ExecInfo()
    name = "h3_seq_to_head" if seq_to_head_dir else "h3_head_to_seq"
    cfg = _config(variant, ctas_per_sm, serial, token_chunks)
    args = [_abi.pointer_array([t.data_ptr() for t in send]),
            _abi.pointer_array([t.data_ptr() for t in recv]),
            T, int(P), int(H), int(D), W, int(window_bytes),
            C.c_void_p(_stream_handle(stream, dev))]
    with _device_guard(dev):
        if cfg is None:
            st = getattr(_abi.lib, name)(*args, C.byref(info))
        else:
            st = getattr(_abi.lib, name + "_ex")(*args, cfg, C.byref(info))
    _abi.check(st, name)
    return info.as_dict()


def seq_to_head(send, recv, *, window_bytes: int = 0, stream=None, variant: int = 0,
                ctas_per_sm: int = 0, serial: bool = False, token_chunks: bool = False) -> dict:
    """Ulysses sequence->head relayout.

    send: W tensors [T_r, P, H, D] (or views of one [T, P, H, D] tensor, see
    ``split_rows``); recv: W tensors [T, P, H_j, D], written.  window_bytes > 0
    moves one plane per launch under that byte bound; with token_chunks=True
    (H3_LAUNCH_CHUNK_TOKENS) the window is cut into token ranges of every
    plane instead, which keeps whole rows together.  serial=True launches in
    plain stream order (H3_LAUNCH_SERIAL) instead of programmatic dependent
    launch.  Returns what ran (launches, chunks, grid, block, variant,
    planes_per_launch)."""
    return _relayout(True, send, recv, window_bytes, stream, variant, ctas_per_sm, serial,
                     token_chunks)


def head_to_seq(send, recv, *, window_bytes: int = 0, stream=None, variant: int = 0,
                ctas_per_sm: int = 0, serial: bool = False, token_chunks: bool = False) -> dict:
    """Inverse head->sequence relayout: send W tensors [T, P, H_j, D] -> recv W
    tensors [T_r, P, H, D].  Options as ``seq_to_head``."""
    return _relayout(False, send, recv, window_bytes, stream, variant, ctas_per_sm, serial,
                     token_chunks)


def ragged_reduce_scatter(partials, bias, out, *, stream=None, ctas_per_sm: int = 0,
                          serial: bool = False) -> dict:
    """Tensor-mode ragged reduce-scatter.

    partials: W BF16 tensors [T, C] (or one [W, T, C] tensor); bias: BF16 [C]
    or None; out: W BF16 tensors [T_r, C], written with
    bf16_rne(((p_0 + p_1) + ... + p_{W-1}) + bias) summed in binary32."""
    partials = _as_list(partials)
    out = _as_list(out)
    W = len(partials)
    if W < 1 or len(out) != W:
        raise ValueError("partials and out need one tensor per rank (same count)")
    tensors = partials + out + ([bias] if bias is not None else [])
    dev = _check_tensors(tensors, "ragged_reduce_scatter")
    if any(t.dtype != torch.bfloat16 for t in tensors):
        raise ValueError("ragged_reduce_scatter works on BF16 tensors")
    if any(t.dim() != 2 for t in partials + out):
        raise ValueError("partials and outputs are 2-D: [tokens, cols]")
    T, Cc = partials[0].shape
    if any(tuple(p.shape) != (T, Cc) for p in partials):
        raise ValueError("all partials must have the same [T, C] shape")
    if bias is not None and tuple(bias.shape) != (Cc,):
        raise ValueError(f"bias must be [C] = [{Cc}]")
    for r, (o, rows) in enumerate(zip(out, _rank_sizes(int(T), W, W)[0])):
        if tuple(o.shape) != (rows, Cc):
            raise ValueError(f"out rank {r}: shape {tuple(o.shape)}, expected {(rows, Cc)}")
    info = ExecInfo()
    cfg = _config(0, ctas_per_sm, serial)
    args = [_abi.pointer_array([p.data_ptr() for p in partials]),
            C.c_void_p(bias.data_ptr() if bias is not None else 0),
            _abi.pointer_array([o.data_ptr() for o in out]),
            int(T), int(Cc), W, C.c_void_p(_stream_handle(stream, dev))]
    with _device_guard(dev):
        if cfg is None:
            st = _abi.lib.h3_ragged_reduce_scatter(*args, C.byref(info))
        else:
            st = _abi.lib.h3_ragged_reduce_scatter_ex(*args, cfg, C.byref(info))
    _abi.check(st, "h3_ragged_reduce_scatter")
    return info.as_dict()


def bulk_wait_timeouts(stream=None, reset: bool = False, device=None) -> int:
    """Expired bounded waits of the bulk relayout kernel on this device
    (``h3_bulk_wait_timeouts``; synchronises the stream).  Non-zero means a
    bulk launch gave up and its output is incomplete."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    count = C.c_uint32(0)
    with _device_guard(dev):
        st = _abi.lib.h3_bulk_wait_timeouts(C.c_void_p(_stream_handle(stream, dev)), C.byref(count),
                                            1 if reset else 0)
    _abi.check(st, "h3_bulk_wait_timeouts")
    return int(count.value)


def bounded_wait_selftest(polls: int, arrive_first: bool, *, stream=None, device=None) -> bool:
    """Run the bulk kernels' bounded barrier wait on a barrier nothing (or one
    arrival) completes (``h3_bounded_wait_selftest``); True if the wait
    expired.  Synchronises the stream."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    expired = C.c_int32(-1)
    with _device_guard(dev):
        st = _abi.lib.h3_bounded_wait_selftest(int(polls), 1 if arrive_first else 0,
                                               C.c_void_p(_stream_handle(stream, dev)),
                                               C.byref(expired))
    _abi.check(st, "h3_bounded_wait_selftest")
    if expired.value not in (0, 1):
        raise RuntimeError("bounded wait self-test did not report")
    return bool(expired.value)


def ragged_all_gather(blocks, out, *, stream=None, variant: int = 0, ctas_per_sm: int = 0,
                      serial: bool = False) -> dict:
    """Ragged all-gather of token rows: blocks are W tensors [T_r, C] (rank
    r's rows; 2-byte elements), out W tensors [T, C], each written with all T
    rows in token order (``h3_ragged_all_gather``)."""
    blocks = _as_list(blocks)
    out = _as_list(out)
    W = len(blocks)
    if W < 1 or len(out) != W:
        raise ValueError("blocks and out need one tensor per rank (same count)")
    dev = _check_tensors(blocks + out, "ragged_all_gather")
    if any(t.dim() != 2 for t in blocks + out):
        raise ValueError("blocks and outputs are 2-D: [tokens, cols]")
    Cc = int(blocks[0].shape[1])
    T = sum(int(b.shape[0]) for b in blocks)
    for r, (b, rows) in enumerate(zip(blocks, _rank_sizes(T, W, W)[0])):
        if tuple(b.shape) != (rows, Cc):
            raise ValueError(f"block {r}: shape {tuple(b.shape)}, expected {(rows, Cc)}")
    for j, o in enumerate(out):
        if tuple(o.shape) != (T, Cc):
            raise ValueError(f"out {j}: shape {tuple(o.shape)}, expected {(T, Cc)}")
    info = ExecInfo()
    args = [_abi.pointer_array([b.data_ptr() for b in blocks]),
            _abi.pointer_array([o.data_ptr() for o in out]),
            T, Cc, W, C.c_void_p(_stream_handle(stream, dev))]
    cfg = _config(variant, ctas_per_sm, serial)
    with _device_guard(dev):
        if cfg is None:
            st = _abi.lib.h3_ragged_all_gather(*args, C.byref(info))
        else:
            st = _abi.lib.h3_ragged_all_gather_ex(*args, cfg, C.byref(info))
    _abi.check(st, "h3_ragged_all_gather")
    return info.as_dict()


def ragged_reduce_scatter_gated(partials, bias, gate, seg_bounds, x, out=None, *,
                                stream=None) -> dict:
    """Ragged reduce-scatter fused with residual gating per packed segment
    (``h3_ragged_reduce_scatter_gated``): out_r = bf16(x_r + gate[seg] * y_r),
    y_r the reduce-scatter output rows of rank r.  gate: BF16 [S, C];
    seg_bounds: S+1 packed segment bounds (0 .. T); x: W tensors [T_r, C];
    out: W tensors [T_r, C], or None to update x in place."""
    partials = _as_list(partials)
    x = _as_list(x)
    out = x if out is None else _as_list(out)
    W = len(partials)
    if W < 1 or len(x) != W or len(out) != W:
        raise ValueError("partials, x and out need one tensor per rank (same count)")
    tensors = partials + x + out + [gate] + ([bias] if bias is not None else [])
    dev = _check_tensors(tensors, "ragged_reduce_scatter_gated")
    if any(t.dtype != torch.bfloat16 for t in tensors):
        raise ValueError("ragged_reduce_scatter_gated works on BF16 tensors")
    T, Cc = partials[0].shape
    b = np.ascontiguousarray(seg_bounds, dtype=np.int64)
    S = len(b) - 1
    if tuple(gate.shape) != (S, Cc):
        raise ValueError(f"gate must be [S, C] = [{S}, {Cc}]")
    for r, rows in enumerate(_rank_sizes(int(T), W, W)[0]):
        for name, t in (("x", x[r]), ("out", out[r])):
            if tuple(t.shape) != (rows, Cc):
                raise ValueError(f"{name} rank {r}: shape {tuple(t.shape)}, expected "
                                 f"{(rows, Cc)}")
    info = ExecInfo()
    with _device_guard(dev):
        st = _abi.lib.h3_ragged_reduce_scatter_gated(
            _abi.pointer_array([p.data_ptr() for p in partials]),
            C.c_void_p(bias.data_ptr() if bias is not None else 0), C.c_void_p(gate.data_ptr()),
            b.ctypes.data_as(_abi._i64p), S,
            _abi.pointer_array([v.data_ptr() for v in x]),
            _abi.pointer_array([o.data_ptr() for o in out]),
            int(T), int(Cc), W, C.c_void_p(_stream_handle(stream, dev)), C.byref(info))
    _abi.check(st, "h3_ragged_reduce_scatter_gated")
    return info.as_dict()


# ---------------------------------------------------------------------------
# prepared calls: validate and marshal once, then one C call per invocation
# ---------------------------------------------------------------------------

# ---------------------------------------------------------------------------
# One rank per GPU: rank k's share of each operation, pulled from every rank's
# buffer (``h3_*_rank``).  Inputs are W tensors or device addresses (for
# example ``peers.PeerBuffers(...).pointers``); the output is this rank's tensor.
# ---------------------------------------------------------------------------
def _addresses(items, what: str) -> list:
    out = []
    for x in items:
        if isinstance(x, torch.Tensor):
            if not x.is_cuda or not x.is_contiguous() or x.element_size() != 2:
                raise ValueError(f"{what}: CUDA, contiguous, 2-byte elements")
            out.append(int(x.data_ptr()))
        elif x is None:
            raise ValueError(f"{what}: no buffer")
        else:
            out.append(int(x))
    return out


def _require_bf16(items, what: str) -> None:
    """The reduce arithmetic reads BF16: refuse tensors of any other 2-byte
    type (device addresses carry no type and are taken as given)."""
    for x in items:
        if isinstance(x, torch.Tensor) and x.dtype != torch.bfloat16:
            raise ValueError(f"{what}: BF16 tensors only (got {x.dtype})")


def _local_output(t: torch.Tensor, what: str, dims: int):
    _check_tensors([t], what)
    if t.dim() != dims:
        raise ValueError(f"{what} must be {dims}-D")
    return t.device


def seq_to_head_rank(send, recv, rank: int, *, n_heads: int, window_bytes: int = 0, stream=None,
                     variant: int = 0, ctas_per_sm: int = 0, serial: bool = False,
                     token_chunks: bool = False) -> dict:
    """Rank ``rank``'s head-side buffer with one rank per GPU
    (``h3_seq_to_head_rank``): send = the W ranks' sequence-side buffers
    [T_r, P, H, D]; recv = this rank's [T, P, H_k, D]."""
    send = list(send)
    W = len(send)
    dev = _local_output(recv, "recv", 4)
    T, P, Hk, D = (int(v) for v in recv.shape)
    if Hk != partition(T, n_heads, W).heads(rank):
        raise ValueError(f"recv has {Hk} heads; rank {rank} of {W} owns "
                         f"{partition(T, n_heads, W).heads(rank)}")
    info = ExecInfo()
    with _device_guard(dev):
        st = _abi.lib.h3_seq_to_head_rank(
            _abi.pointer_array(_addresses(send, "send")), C.c_void_p(recv.data_ptr()), T, P,
            int(n_heads), D, W, int(rank), int(window_bytes),
            C.c_void_p(_stream_handle(stream, dev)),
            _config(variant, ctas_per_sm, serial, token_chunks), C.byref(info))
    _abi.check(st, "h3_seq_to_head_rank")
    return info.as_dict()


def head_to_seq_rank(send, recv, rank: int, *, n_tokens: int, window_bytes: int = 0, stream=None,
                     variant: int = 0, ctas_per_sm: int = 0, serial: bool = False,
                     token_chunks: bool = False) -> dict:
    """Rank ``rank``'s sequence-side rows with one rank per GPU
    (``h3_head_to_seq_rank``): send = the W ranks' head-side buffers
    [T, P, H_j, D]; recv = this rank's [T_k, P, H, D]."""
    send = list(send)
    W = len(send)
    dev = _local_output(recv, "recv", 4)
    Tk, P, H, D = (int(v) for v in recv.shape)
    if Tk != partition(n_tokens, H, W).tokens(rank):
        raise ValueError(f"recv has {Tk} tokens; rank {rank} of {W} owns "
                         f"{partition(n_tokens, H, W).tokens(rank)}")
    info = ExecInfo()
    with _device_guard(dev):
        st = _abi.lib.h3_head_to_seq_rank(
            _abi.pointer_array(_addresses(send, "send")), C.c_void_p(recv.data_ptr()),
            int(n_tokens), P, H, D, W, int(rank), int(window_bytes),
            C.c_void_p(_stream_handle(stream, dev)),
            _config(variant, ctas_per_sm, serial, token_chunks), C.byref(info))
    _abi.check(st, "h3_head_to_seq_rank")
    return info.as_dict()


def ragged_reduce_scatter_rank(partials, bias, out, rank: int, *, n_tokens: int, stream=None,
                               ctas_per_sm: int = 0, serial: bool = False) -> dict:
    """Rank ``rank``'s rows of the ragged reduce-scatter with one rank per GPU
    (``h3_ragged_reduce_scatter_rank``): partials = the W ranks' [T, C];
    bias = [C] tensor, address or None; out = this rank's [T_k, C]."""
    partials = list(partials)
    W = len(partials)
    dev = _local_output(out, "out", 2)
    _require_bf16(partials + [bias, out], "ragged_reduce_scatter_rank")
    Tk, Cc = (int(v) for v in out.shape)
    if Tk != partition(n_tokens, W, W).tokens(rank):
        raise ValueError(f"out has {Tk} rows; rank {rank} of {W} owns "
                         f"{partition(n_tokens, W, W).tokens(rank)}")
    b = 0 if bias is None else _addresses([bias], "bias")[0]
    info = ExecInfo()
    with _device_guard(dev):
        st = _abi.lib.h3_ragged_reduce_scatter_rank(
            _abi.pointer_array(_addresses(partials, "partials")), C.c_void_p(b),
            C.c_void_p(out.data_ptr()), int(n_tokens), Cc, W, int(rank),
            C.c_void_p(_stream_handle(stream, dev)), _config(0, ctas_per_sm, serial),
            C.byref(info))
    _abi.check(st, "h3_ragged_reduce_scatter_rank")
    return info.as_dict()


def ragged_reduce_scatter_gated_rank(partials, bias, gate, seg_bounds, x, rank: int, *,
                                     n_tokens: int, out=None, stream=None,
                                     serial: bool = False) -> dict:
    """Rank ``rank``'s rows of the gated reduce-scatter with one rank per GPU
    (``h3_ragged_reduce_scatter_gated_rank``): partials = the W ranks' [T, C];
    gate [S, C] and bias [C] (tensors or addresses); seg_bounds = the S+1
    global packed bounds; x = this rank's residual [T_k, C]; out = x (in
    place) unless given."""
    partials = list(partials)
    W = len(partials)
    dev = _local_output(x, "x", 2)
    out = x if out is None else out
    _local_output(out, "out", 2)
    _require_bf16(partials + [bias, gate, x, out], "ragged_reduce_scatter_gated_rank")
    Tk, Cc = (int(v) for v in x.shape)
    if tuple(out.shape) != (Tk, Cc):
        raise ValueError("out must have x's shape")
    if Tk != partition(n_tokens, W, W).tokens(rank):
        raise ValueError(f"x has {Tk} rows; rank {rank} of {W} owns "
                         f"{partition(n_tokens, W, W).tokens(rank)}")
    bounds = np.ascontiguousarray(np.asarray(seg_bounds, dtype=np.int64))
    b = 0 if bias is None else _addresses([bias], "bias")[0]
    info = ExecInfo()
    with _device_guard(dev):
        st = _abi.lib.h3_ragged_reduce_scatter_gated_rank(
            _abi.pointer_array(_addresses(partials, "partials")), C.c_void_p(b),
            C.c_void_p(_addresses([gate], "gate")[0]),
            bounds.ctypes.data_as(C.POINTER(C.c_int64)), int(bounds.size - 1),
            C.c_void_p(x.data_ptr()), C.c_void_p(out.data_ptr()), int(n_tokens), Cc, W, int(rank),
            C.c_void_p(_stream_handle(stream, dev)), _config(0, 0, serial), C.byref(info))
    _abi.check(st, "h3_ragged_reduce_scatter_gated_rank")
    return info.as_dict()


def ragged_all_gather_rank(blocks, out, rank: int, *, stream=None, ctas_per_sm: int = 0,
                           serial: bool = False) -> dict:
    """Rank ``rank``'s copy of the ragged all-gather with one rank per GPU
    (``h3_ragged_all_gather_rank``): blocks = the W ranks' [T_r, C]; out =
    this rank's [T, C]."""
    blocks = list(blocks)
    W = len(blocks)
    dev = _local_output(out, "out", 2)
    T, Cc = (int(v) for v in out.shape)
    info = ExecInfo()
    with _device_guard(dev):
        st = _abi.lib.h3_ragged_all_gather_rank(
            _abi.pointer_array(_addresses(blocks, "blocks")), C.c_void_p(out.data_ptr()), T, Cc,
            W, int(rank), C.c_void_p(_stream_handle(stream, dev)),
            _config(0, ctas_per_sm, serial), C.byref(info))
    _abi.check(st, "h3_ragged_all_gather_rank")
    return info.as_dict()


class PreparedRelayout:
    """A relayout whose shapes, buffers and launch options are checked and
    marshalled once; calling it issues one C call (``h3_*_layout``) on the
    given (or current) stream.  The buffers are captured by address: refill
    them in place between calls, do not replace them.

    ``inverse(send, recv)`` prepares the opposite direction over the same
    shapes (FastVideo PR #1807, "Problem and behavior": the backward pass
    reuses the plan saved by its forward)."""

    def __init__(self, seq_to_head_dir: bool, send, recv, *, layout: int = 0,
                 window_bytes: int = 0, variant: int = 0, ctas_per_sm: int = 0,
                 serial: bool = False, token_chunks: bool = False):
        send = _as_list(send)
        recv = _as_list(recv)
        T, P, H, D, W, dev = _relayout_shapes(seq_to_head_dir, send, recv, layout)
        self.seq_to_head_dir = seq_to_head_dir
        self.shape = (T, P, H, D, W)
        self.device = dev
        self.layout = int(layout)
        self.window_bytes = int(window_bytes)
        self.variant = int(variant)
        self.ctas_per_sm = int(ctas_per_sm)
        self.serial = bool(serial)
        self.token_chunks = bool(token_chunks)
        self._keep = (send, recv)  # keep the tensors alive while the call holds their addresses
        name = "h3_seq_to_head_layout" if seq_to_head_dir else "h3_head_to_seq_layout"
        self._fn = getattr(_abi.lib, name)
        self._name = name
        self._cfg = LaunchConfig(self.variant, self.ctas_per_sm,
                                 _flags(self.serial, self.token_chunks), 0)
        self._info = ExecInfo()
        self._head = (_abi.pointer_array([t.data_ptr() for t in send]),
                      _abi.pointer_array([t.data_ptr() for t in recv]),
                      T, P, H, D, W, self.window_bytes, self.layout)

    def __call__(self, stream=None) -> ExecInfo:
        s = self.device_stream(stream)
        st = self._fn(*self._head, s, C.byref(self._cfg), C.byref(self._info))
        if st != _abi.H3_OK:
            raise H3Error(st, self._name)
        return self._info

    def device_stream(self, stream):
        """The cudaStream_t to launch on: `stream`, or the current stream of
        the prepared call's device."""
        if stream is None:
            return C.c_void_p(torch.cuda.current_stream(self.device).cuda_stream)
        return C.c_void_p(_stream_handle(stream, self.device))

    def inverse(self, send, recv) -> "PreparedRelayout":
        """The opposite direction with the same layout, window and launch
        options; send/recv are that direction's buffers."""
        return PreparedRelayout(not self.seq_to_head_dir, send, recv, layout=self.layout,
                                window_bytes=self.window_bytes, variant=self.variant,
                                ctas_per_sm=self.ctas_per_sm, serial=self.serial,
                                token_chunks=self.token_chunks)


def prepare_seq_to_head(send, recv, **kw) -> PreparedRelayout:
    """Prepared ``seq_to_head`` / ``seq_to_head_layout`` (see ``PreparedRelayout``)."""
    return PreparedRelayout(True, send, recv, **kw)


def prepare_head_to_seq(send, recv, **kw) -> PreparedRelayout:
    """Prepared ``head_to_seq`` / ``head_to_seq_layout`` (see ``PreparedRelayout``)."""
    return PreparedRelayout(False, send, recv, **kw)


class PreparedReduceScatter:
    """A ragged reduce-scatter checked and marshalled once; each call is one
    ``h3_ragged_reduce_scatter_ex`` call.  Buffers are captured by address."""

    def __init__(self, partials, bias, out, *, ctas_per_sm: int = 0, serial: bool = False):
        partials = _as_list(partials)
        out = _as_list(out)
        W = len(partials)
        tensors = partials + out + ([bias] if bias is not None else [])
        self.device = _check_tensors(tensors, "ragged_reduce_scatter")
        if any(t.dtype != torch.bfloat16 for t in tensors):
            raise ValueError("ragged_reduce_scatter works on BF16 tensors")
        T, Cc = partials[0].shape
        if any(tuple(p.shape) != (T, Cc) for p in partials) or len(out) != W:
            raise ValueError("partials must share one [T, C] shape, one output per rank")
        part = partition(T, W, W)
        for r, o in enumerate(out):
            if tuple(o.shape) != (part.tokens(r), Cc):
                raise ValueError(f"out rank {r}: shape {tuple(o.shape)}, expected {(part.tokens(r), Cc)}")
        self._keep = (partials, bias, out)
        self._cfg = LaunchConfig(0, int(ctas_per_sm), H3_LAUNCH_SERIAL if serial else 0, 0)
        self._info = ExecInfo()
        self._head = (_abi.pointer_array([p.data_ptr() for p in partials]),
                      C.c_void_p(bias.data_ptr() if bias is not None else 0),
                      _abi.pointer_array([o.data_ptr() for o in out]), int(T), int(Cc), W)

    def __call__(self, stream=None) -> ExecInfo:
        s = C.c_void_p(_stream_handle(stream, self.device))
        st = _abi.lib.h3_ragged_reduce_scatter_ex(*self._head, s, C.byref(self._cfg), C.byref(self._info))
        if st != _abi.H3_OK:
            raise H3Error(st, "h3_ragged_reduce_scatter")
        return self._info


def prepare_ragged_reduce_scatter(partials, bias, out, **kw) -> PreparedReduceScatter:
    """A reduce-scatter over fixed buffers, checked and marshalled once;
    calling it issues one C call (same arguments as ``ragged_reduce_scatter``)."""
    return PreparedReduceScatter(partials, bias, out, **kw)


def alloc_reduce_outputs(T: int, C_: int, W: int, device, dtype=torch.bfloat16):
    """One [T, C] tensor and its per-rank [T_r, C] row views."""
    part = partition(T, W, W)
    full = torch.empty((T, C_), dtype=dtype, device=device)
    return full, split_rows(full, part.token_starts)
