"""ctypes declarations of ``include/h3rr.h`` and loading of ``libh3rr.so``.

The shared library is built in-tree (``ragged_reduce_b200/build.py``).  There
is no fallback: if the library is missing or cannot be loaded, importing the
package raises.
"""
from __future__ import annotations

import ctypes as C
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libh3rr.so")
HEADER_PATH = os.path.join(os.path.dirname(PKG), "include", "h3rr.h")

H3_OK = 0
H3_ERR_INVALID_ARG = 1
H3_ERR_EMPTY_PARTITION = 2
H3_ERR_MISALIGNED = 3
H3_ERR_WINDOW = 4
H3_ERR_UNSUPPORTED = 5
H3_ERR_CUDA = 6

STATUS_NAMES = {
    H3_OK: "H3_OK",
    H3_ERR_INVALID_ARG: "H3_ERR_INVALID_ARG",
    H3_ERR_EMPTY_PARTITION: "H3_ERR_EMPTY_PARTITION",
    H3_ERR_MISALIGNED: "H3_ERR_MISALIGNED",
    H3_ERR_WINDOW: "H3_ERR_WINDOW",
    H3_ERR_UNSUPPORTED: "H3_ERR_UNSUPPORTED",
    H3_ERR_CUDA: "H3_ERR_CUDA",
}

H3_VARIANT_NONE = 0
H3_VARIANT_VECTOR = 1
H3_VARIANT_BULK = 2
H3_VARIANT_REDUCE = 3
H3_VARIANT_STAGED = 4
H3_VARIANT_GATHER = 5
H3_VARIANT_REDUCE_GATED = 6
MAX_GATE_SEGMENTS = 256

MAX_WORLD = 64
H3_LAYOUT_SEQ_PLANE_MAJOR = 1
H3_LAYOUT_HEAD_PLANE_MAJOR = 2
H3_LAUNCH_SERIAL = 1
H3_LAUNCH_CHUNK_TOKENS = 2
H3_IPC_HANDLE_BYTES = 64
ABI_VERSION = 3


class ExecInfo(C.Structure):
    _fields_ = [
        ("launches", C.c_int32),
        ("chunks", C.c_int32),
        ("grid", C.c_int32),
        ("block", C.c_int32),
        ("variant", C.c_int32),
        ("planes_per_launch", C.c_int32),
    ]

    def as_dict(self) -> dict:
        return {name: int(getattr(self, name)) for name, _ in self._fields_}


class LaunchConfig(C.Structure):
    _fields_ = [
        ("variant", C.c_int32),
        ("ctas_per_sm", C.c_int32),
        ("flags", C.c_int32),
        ("reserved1", C.c_int32),
    ]


class IpcHandle(C.Structure):
    _fields_ = [
        ("handle", C.c_ubyte * H3_IPC_HANDLE_BYTES),
        ("offset", C.c_int64),
        ("alloc_bytes", C.c_int64),
    ]


class H3Error(RuntimeError):
    """A non-OK status from the C ABI."""

    def __init__(self, status: int, call: str):
        self.status = int(status)
        self.call = call
        name = STATUS_NAMES.get(self.status, str(self.status))
        detail = ""
        self.cuda_error = 0
        if self.status == H3_ERR_CUDA:
            msg = C.c_char_p()
            self.cuda_error = int(lib.h3_last_cuda_error(C.byref(msg)))
            detail = f"; cudaError {self.cuda_error}: {msg.value.decode() if msg.value else ''}"
        super().__init__(f"{call}: {name} ({describe(self.status)}{detail})")


_i64p = C.POINTER(C.c_int64)
_i32p = C.POINTER(C.c_int32)
_vpp = C.POINTER(C.c_void_p)

_RELAYOUT_ARGS = [_vpp, _vpp, C.c_int64, C.c_int32, C.c_int32, C.c_int32, C.c_int32,
                  C.c_int64, C.c_void_p]
_REDUCE_ARGS = [_vpp, C.c_void_p, _vpp, C.c_int64, C.c_int64, C.c_int32, C.c_void_p]


def _load() -> C.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"ragged_reduce_b200: CUDA library not built ({LIB_PATH} missing); "
            "run `python ragged_reduce_b200/build.py` or __graft_entry__.build()")
    lib = C.CDLL(LIB_PATH)
    lib.h3_abi_version.restype = C.c_int32
    lib.h3_abi_version.argtypes = []
    lib.h3_status_string.restype = C.c_char_p
    lib.h3_status_string.argtypes = [C.c_int]
    lib.h3_partition.restype = C.c_int
    lib.h3_partition.argtypes = [C.c_int64, C.c_int32, C.c_int32, _i64p, C.c_int32, _i64p,
                                 _i32p, _i64p, _i32p, _i32p]
    for name in ("h3_seq_to_head", "h3_head_to_seq"):
        f = getattr(lib, name)
        f.restype = C.c_int
        f.argtypes = _RELAYOUT_ARGS + [C.POINTER(ExecInfo)]
        fx = getattr(lib, name + "_ex")
        fx.restype = C.c_int
        fx.argtypes = _RELAYOUT_ARGS + [C.POINTER(LaunchConfig), C.POINTER(ExecInfo)]
    lib.h3_ragged_reduce_scatter.restype = C.c_int
    lib.h3_ragged_reduce_scatter.argtypes = _REDUCE_ARGS + [C.POINTER(ExecInfo)]
    lib.h3_ragged_reduce_scatter_ex.restype = C.c_int
    lib.h3_ragged_reduce_scatter_ex.argtypes = _REDUCE_ARGS + [C.POINTER(LaunchConfig),
                                                               C.POINTER(ExecInfo)]
    for name in ("h3_seq_to_head_staged", "h3_head_to_seq_staged"):
        f = getattr(lib, name)
        f.restype = C.c_int
        f.argtypes = [_vpp, _vpp, C.c_int64, C.c_int32, C.c_int32, C.c_int32, C.c_int32,
                      C.c_void_p, C.c_int64, C.c_void_p, C.POINTER(ExecInfo)]
    for name in ("h3_seq_to_head_layout", "h3_head_to_seq_layout"):
        f = getattr(lib, name)
        f.restype = C.c_int
        f.argtypes = [_vpp, _vpp, C.c_int64, C.c_int32, C.c_int32, C.c_int32, C.c_int32,
                      C.c_int64, C.c_int32, C.c_void_p, C.POINTER(LaunchConfig),
                      C.POINTER(ExecInfo)]
    lib.h3_ragged_all_gather.restype = C.c_int
    lib.h3_ragged_all_gather.argtypes = [_vpp, _vpp, C.c_int64, C.c_int64, C.c_int32, C.c_void_p,
                                         C.POINTER(ExecInfo)]
    lib.h3_ragged_all_gather_ex.restype = C.c_int
    lib.h3_ragged_all_gather_ex.argtypes = [_vpp, _vpp, C.c_int64, C.c_int64, C.c_int32,
                                            C.c_void_p, C.POINTER(LaunchConfig),
                                            C.POINTER(ExecInfo)]
    lib.h3_ragged_reduce_scatter_gated.restype = C.c_int
    lib.h3_ragged_reduce_scatter_gated.argtypes = [_vpp, C.c_void_p, C.c_void_p, _i64p, C.c_int32,
                                                   _vpp, _vpp, C.c_int64, C.c_int64, C.c_int32,
                                                   C.c_void_p, C.POINTER(ExecInfo)]
    lib.h3_staged_plan.restype = C.c_int
    lib.h3_staged_plan.argtypes = [C.c_int64, C.c_int32, C.c_int32, C.c_int32, C.c_int64,
                                   _i64p, _i64p]
    lib.h3_relayout_chunk_plan.restype = C.c_int
    lib.h3_relayout_chunk_plan.argtypes = [C.c_int64, C.c_int32, C.c_int32, C.c_int32, C.c_int32,
                                           C.c_int64, _i64p, _i64p]
    lib.h3_relayout_chunk_plan_ex.restype = C.c_int
    lib.h3_relayout_chunk_plan_ex.argtypes = [C.c_int64, C.c_int32, C.c_int32, C.c_int32, C.c_int32,
                                              C.c_int64, C.c_int32, _i64p, _i64p,
                                              C.POINTER(C.c_int32)]
    lib.h3_last_cuda_error.restype = C.c_int32
    lib.h3_last_cuda_error.argtypes = [C.POINTER(C.c_char_p)]
    lib.h3_bulk_wait_timeouts.restype = C.c_int
    lib.h3_bulk_wait_timeouts.argtypes = [C.c_void_p, C.POINTER(C.c_uint32), C.c_int32]
    for name in ("h3_seq_to_head_rank", "h3_head_to_seq_rank"):
        f = getattr(lib, name)
        f.restype = C.c_int
        f.argtypes = [_vpp, C.c_void_p, C.c_int64, C.c_int32, C.c_int32, C.c_int32, C.c_int32,
                      C.c_int32, C.c_int64, C.c_void_p, C.POINTER(LaunchConfig),
                      C.POINTER(ExecInfo)]
    lib.h3_ragged_reduce_scatter_rank.restype = C.c_int
    lib.h3_ragged_reduce_scatter_rank.argtypes = [_vpp, C.c_void_p, C.c_void_p, C.c_int64,
                                                  C.c_int64, C.c_int32, C.c_int32, C.c_void_p,
                                                  C.POINTER(LaunchConfig), C.POINTER(ExecInfo)]
    lib.h3_ragged_reduce_scatter_gated_rank.restype = C.c_int
    lib.h3_ragged_reduce_scatter_gated_rank.argtypes = [
        _vpp, C.c_void_p, C.c_void_p, _i64p, C.c_int32, C.c_void_p, C.c_void_p, C.c_int64,
        C.c_int64, C.c_int32, C.c_int32, C.c_void_p, C.POINTER(LaunchConfig), C.POINTER(ExecInfo)]
    lib.h3_ragged_all_gather_rank.restype = C.c_int
    lib.h3_ragged_all_gather_rank.argtypes = [_vpp, C.c_void_p, C.c_int64, C.c_int64, C.c_int32,
                                              C.c_int32, C.c_void_p, C.POINTER(LaunchConfig),
                                              C.POINTER(ExecInfo)]
    lib.h3_bounded_wait_selftest.restype = C.c_int
    lib.h3_bounded_wait_selftest.argtypes = [C.c_uint32, C.c_int32, C.c_void_p,
                                             C.POINTER(C.c_int32)]
    lib.h3_ipc_export.restype = C.c_int
    lib.h3_ipc_export.argtypes = [C.c_void_p, C.POINTER(IpcHandle)]
    lib.h3_ipc_open.restype = C.c_int
    lib.h3_ipc_open.argtypes = [C.POINTER(IpcHandle), C.POINTER(C.c_void_p)]
    lib.h3_ipc_close.restype = C.c_int
    lib.h3_ipc_close.argtypes = [C.c_void_p, C.POINTER(IpcHandle)]
    version = lib.h3_abi_version()
    if version != ABI_VERSION:
        raise ImportError(f"libh3rr ABI version {version}, binding expects {ABI_VERSION}")
    return lib


lib = _load()


def describe(status: int) -> str:
    s = lib.h3_status_string(int(status))
    return s.decode() if s else "unknown"


def check(status: int, call: str) -> None:
    if status != H3_OK:
        raise H3Error(status, call)


def pointer_array(ptrs) -> C.Array:
    return (C.c_void_p * len(ptrs))(*ptrs)
