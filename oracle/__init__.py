"""Plain CPU oracle for the H3 Ulysses relayouts and the ragged reduce-scatter.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference arm of ``bench.py`` may import this package.  The
product library (``ragged_reduce_b200``) never imports, links or calls it, and
this package never imports the product library: the two share no code.

The arithmetic lives in ``h3_oracle.c`` (plain C99, scalar loops, written from
the pages' definitions; see the header of that file for the citations).  This
module is ctypes marshalling of numpy arrays only.  BF16 tensors travel as
``numpy.uint16`` arrays of their raw bit patterns.
"""
from __future__ import annotations

import ctypes as C

import numpy as np

from . import build as _build

_u16p = C.POINTER(C.c_uint16)
_i64p = C.POINTER(C.c_int64)
_i32p = C.POINTER(C.c_int32)
_f32p = C.POINTER(C.c_float)


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctype)


def _ptr_array(arrays):
    arr = (C.c_void_p * len(arrays))()
    for i, a in enumerate(arrays):
        arr[i] = a.ctypes.data
    return arr


class Oracle:
    """ctypes view of one compiled copy of the oracle."""

    def __init__(self, lib_path: str):
        lib = C.CDLL(lib_path)
        lib.h3o_bf16_to_f32.restype = C.c_float
        lib.h3o_bf16_to_f32.argtypes = [C.c_uint16]
        lib.h3o_f32_to_bf16_rne.restype = C.c_uint16
        lib.h3o_f32_to_bf16_rne.argtypes = [C.c_float]
        lib.h3o_bf16_to_f32_array.argtypes = [_u16p, _f32p, C.c_int64]
        lib.h3o_f32_to_bf16_array.argtypes = [_f32p, _u16p, C.c_int64]
        lib.h3o_partition_range.restype = C.c_int32
        lib.h3o_partition_range.argtypes = [C.c_int64, C.c_int32, _i64p]
        lib.h3o_owner.restype = C.c_int32
        lib.h3o_owner.argtypes = [_i64p, C.c_int32, C.c_int64]
        lib.h3o_clip_segments.restype = C.c_int32
        lib.h3o_clip_segments.argtypes = [_i64p, C.c_int32, C.c_int64, C.c_int64, _i64p, _i32p]
        for name in ("h3o_seq_to_head", "h3o_head_to_seq"):
            f = getattr(lib, name)
            f.restype = C.c_int32
            f.argtypes = [C.c_void_p, C.c_void_p, C.c_int64, C.c_int32, C.c_int32,
                          C.c_int32, C.c_int32]
        for name in ("h3o_seq_to_head_locate", "h3o_head_to_seq_locate"):
            f = getattr(lib, name)
            f.restype = C.c_int32
            f.argtypes = [C.c_int64, C.c_int32, C.c_int32, C.c_int32, C.c_int32,
                          C.c_int32, C.c_int64, _i64p, _i32p, _i64p]
        lib.h3o_reduce_scatter_gated.restype = C.c_int32
        lib.h3o_reduce_scatter_gated.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p, _i64p,
                                                 C.c_int32, C.c_void_p, C.c_void_p, C.c_int64,
                                                 C.c_int64, C.c_int32]
        lib.h3o_relayout_layout.restype = C.c_int32
        lib.h3o_relayout_layout.argtypes = [C.c_void_p, C.c_void_p, C.c_int64, C.c_int32,
                                            C.c_int32, C.c_int32, C.c_int32, C.c_int32,
                                            C.c_int32, C.c_int32]
        lib.h3o_ragged_all_gather.restype = C.c_int32
        lib.h3o_ragged_all_gather.argtypes = [C.c_void_p, C.c_void_p, C.c_int64, C.c_int64,
                                              C.c_int32]
        lib.h3o_reduce_rows.restype = None
        lib.h3o_reduce_rows.argtypes = [C.c_void_p, C.c_void_p, _u16p, C.c_int64,
                                        C.c_int64, C.c_int32]
        lib.h3o_ragged_reduce_scatter.restype = C.c_int32
        lib.h3o_ragged_reduce_scatter.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p,
                                                  C.c_int64, C.c_int64, C.c_int32]
        self.lib = lib
        self.path = lib_path

    # -- BF16 conversions ---------------------------------------------------
    def bf16_to_f32(self, bits) -> np.ndarray:
        a = np.ascontiguousarray(bits, dtype=np.uint16)
        out = np.empty(a.shape, dtype=np.float32)
        self.lib.h3o_bf16_to_f32_array(_ptr(a, _u16p), _ptr(out, _f32p), a.size)
        return out

    def f32_to_bf16(self, x) -> np.ndarray:
        a = np.ascontiguousarray(x, dtype=np.float32)
        out = np.empty(a.shape, dtype=np.uint16)
        self.lib.h3o_f32_to_bf16_array(_ptr(a, _f32p), _ptr(out, _u16p), a.size)
        return out

    # -- partition contract ---------------------------------------------------
    def partition_range(self, n: int, w: int) -> np.ndarray:
        starts = np.zeros(max(w, 0) + 1, dtype=np.int64)
        if self.lib.h3o_partition_range(n, w, _ptr(starts, _i64p)) != 0:
            raise ValueError(f"empty partition: n={n} over w={w}")
        return starts

    def owner(self, starts: np.ndarray, x: int) -> int:
        s = np.ascontiguousarray(starts, dtype=np.int64)
        return int(self.lib.h3o_owner(_ptr(s, _i64p), len(s) - 1, x))

    def clip_segments(self, bounds, ts: int, te: int):
        """Pieces of the packed segments inside [ts, te), rebased to ts.

        Returns (local_bounds int64 [n+1], seg_ids int32 [n])."""
        b = np.ascontiguousarray(bounds, dtype=np.int64)
        n_segs = len(b) - 1
        lb = np.zeros(n_segs + 1, dtype=np.int64)
        ids = np.zeros(max(n_segs, 1), dtype=np.int32)
        n = self.lib.h3o_clip_segments(_ptr(b, _i64p), n_segs, ts, te,
                                       _ptr(lb, _i64p), _ptr(ids, _i32p))
        return lb[: n + 1].copy(), ids[:n].copy()

    # -- relayouts --------------------------------------------------------------
    def seq_to_head(self, send, T: int, P: int, H: int, D: int, W: int):
        """send: W uint16 arrays [T_r, P, H, D] -> W arrays [T, P, H_j, D]."""
        ts = self.partition_range(T, W)
        hs = self.partition_range(H, W)
        src = [np.ascontiguousarray(s, dtype=np.uint16) for s in send]
        for r, s in enumerate(src):
            assert s.size == (ts[r + 1] - ts[r]) * P * H * D
        out = [np.zeros((T, P, int(hs[j + 1] - hs[j]), D), dtype=np.uint16) for j in range(W)]
        rc = self.lib.h3o_seq_to_head(_ptr_array(src), _ptr_array(out), T, P, H, D, W)
        assert rc == 0
        return out

    def head_to_seq(self, send, T: int, P: int, H: int, D: int, W: int):
        """send: W uint16 arrays [T, P, H_j, D] -> W arrays [T_r, P, H, D]."""
        ts = self.partition_range(T, W)
        hs = self.partition_range(H, W)
        src = [np.ascontiguousarray(s, dtype=np.uint16) for s in send]
        for j, s in enumerate(src):
            assert s.size == T * P * (hs[j + 1] - hs[j]) * D
        out = [np.zeros((int(ts[r + 1] - ts[r]), P, H, D), dtype=np.uint16) for r in range(W)]
        rc = self.lib.h3o_head_to_seq(_ptr_array(src), _ptr_array(out), T, P, H, D, W)
        assert rc == 0
        return out

    def _locate(self, fn, T, P, H, D, W, rank, out_elem):
        e = np.ascontiguousarray(out_elem, dtype=np.int64)
        src_rank = np.empty(e.shape, dtype=np.int32)
        src_elem = np.empty(e.shape, dtype=np.int64)
        rc = fn(T, P, H, D, W, rank, e.size, _ptr(e, _i64p), _ptr(src_rank, _i32p),
                _ptr(src_elem, _i64p))
        if rc != 0:
            raise ValueError("locate: bad partition or element index out of range")
        return src_rank, src_elem

    def seq_to_head_locate(self, T, P, H, D, W, j, out_elem):
        """Element indices of head-side rank j's buffer -> (source seq rank, element)."""
        return self._locate(self.lib.h3o_seq_to_head_locate, T, P, H, D, W, j, out_elem)

    def head_to_seq_locate(self, T, P, H, D, W, r, out_elem):
        """Element indices of seq-side rank r's buffer -> (source head rank, element)."""
        return self._locate(self.lib.h3o_head_to_seq_locate, T, P, H, D, W, r, out_elem)

    # -- reduce-scatter ---------------------------------------------------------
    def reduce_rows(self, partials, bias):
        """partials: W uint16 arrays [rows, C]; bias uint16 [C] or None -> [rows, C]."""
        src = [np.ascontiguousarray(p, dtype=np.uint16) for p in partials]
        rows, cols = src[0].shape
        for p in src:
            assert p.shape == (rows, cols)
        b = None if bias is None else np.ascontiguousarray(bias, dtype=np.uint16)
        out = np.zeros((rows, cols), dtype=np.uint16)
        self.lib.h3o_reduce_rows(_ptr_array(src), None if b is None else b.ctypes.data,
                                 _ptr(out, _u16p), rows, cols, len(src))
        return out

    def ragged_reduce_scatter(self, partials, bias, W: int):
        """partials: W uint16 arrays [T, C]; bias [C] or None -> W arrays [T_r, C]."""
        src = [np.ascontiguousarray(p, dtype=np.uint16) for p in partials]
        assert len(src) == W
        T, Cc = src[0].shape
        ts = self.partition_range(T, W)
        b = None if bias is None else np.ascontiguousarray(bias, dtype=np.uint16)
        out = [np.zeros((int(ts[r + 1] - ts[r]), Cc), dtype=np.uint16) for r in range(W)]
        rc = self.lib.h3o_ragged_reduce_scatter(_ptr_array(src),
                                                None if b is None else b.ctypes.data,
                                                _ptr_array(out), T, Cc, W)
        assert rc == 0
        return out

    def relayout_layout(self, send, T, P, H, D, W, seq_to_head: bool, seq_plane_major: bool,
                        head_plane_major: bool):
        """Relayout with plane-major options.  seq_to_head: send are W sequence-side
        buffers ([T_r, P, H, D] or [P, T_r, H, D]) -> W head-side buffers ([T, P, H_j, D]
        or [P, T, H_j, D]); otherwise the reverse."""
        ts = self.partition_range(T, W)
        hs = self.partition_range(H, W)
        src = [np.ascontiguousarray(s, dtype=np.uint16) for s in send]

        def seq_shape(r):
            Tr = int(ts[r + 1] - ts[r])
            return (P, Tr, H, D) if seq_plane_major else (Tr, P, H, D)

        def head_shape(j):
            Hj = int(hs[j + 1] - hs[j])
            return (P, T, Hj, D) if head_plane_major else (T, P, Hj, D)

        if seq_to_head:
            for r, x in enumerate(src):
                assert x.size == int(np.prod(seq_shape(r)))
            out = [np.zeros(head_shape(j), dtype=np.uint16) for j in range(W)]
        else:
            for j, x in enumerate(src):
                assert x.size == int(np.prod(head_shape(j)))
            out = [np.zeros(seq_shape(r), dtype=np.uint16) for r in range(W)]
        rc = self.lib.h3o_relayout_layout(_ptr_array(src), _ptr_array(out), T, P, H, D, W,
                                          1 if seq_to_head else 0, int(seq_plane_major),
                                          int(head_plane_major))
        assert rc == 0
        return out

    def reduce_scatter_gated(self, partials, bias, gate, bounds, x, W: int):
        """partials: W uint16 [T, C]; bias [C] or None; gate [S, C]; bounds int64 [S+1];
        x: W uint16 [T_r, C] -> W arrays [T_r, C] = bf16(x + gate[seg] * reduce-scatter)."""
        src = [np.ascontiguousarray(p, dtype=np.uint16) for p in partials]
        assert len(src) == W
        T, Cc = src[0].shape
        ts = self.partition_range(T, W)
        xs = [np.ascontiguousarray(v, dtype=np.uint16) for v in x]
        for r, v in enumerate(xs):
            assert v.shape == (ts[r + 1] - ts[r], Cc)
        b = None if bias is None else np.ascontiguousarray(bias, dtype=np.uint16)
        g = np.ascontiguousarray(gate, dtype=np.uint16)
        bd = np.ascontiguousarray(bounds, dtype=np.int64)
        S = len(bd) - 1
        assert g.shape == (S, Cc)
        out = [np.zeros_like(v) for v in xs]
        rc = self.lib.h3o_reduce_scatter_gated(_ptr_array(src), None if b is None else b.ctypes.data,
                                               g.ctypes.data, _ptr(bd, _i64p), S, _ptr_array(xs),
                                               _ptr_array(out), T, Cc, W)
        assert rc == 0
        return out

    def ragged_all_gather(self, blocks, W: int):
        """blocks: W uint16 arrays [T_r, C] -> W arrays [T, C] (every rank gets all rows)."""
        src = [np.ascontiguousarray(b, dtype=np.uint16) for b in blocks]
        assert len(src) == W
        Cc = src[0].shape[1]
        T = sum(b.shape[0] for b in src)
        ts = self.partition_range(T, W)
        for r, b in enumerate(src):
            assert b.shape == (ts[r + 1] - ts[r], Cc)
        out = [np.zeros((T, Cc), dtype=np.uint16) for _ in range(W)]
        rc = self.lib.h3o_ragged_all_gather(_ptr_array(src), _ptr_array(out), T, Cc, W)
        assert rc == 0
        return out


_default: Oracle | None = None


def load(lib_path: str | None = None) -> Oracle:
    """The oracle compiled from ``h3_oracle.c`` (built with gcc when stale)."""
    global _default
    if lib_path is not None:
        return Oracle(lib_path)
    if _default is None:
        if _build.is_stale():
            _build.build()
        _default = Oracle(_build.LIB)
    return _default


def __getattr__(name):
    # Module-level shortcuts: oracle.seq_to_head(...) etc. use the default build.
    if name.startswith("_"):
        raise AttributeError(name)
    return getattr(load(), name)


LIB_PATH = _build.LIB
SRC_PATH = _build.SRC
