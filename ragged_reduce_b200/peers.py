"""Every rank's buffer, addressable from this process (one rank per GPU).

The ``*_rank`` calls take the W ranks' input buffers as device addresses the
local GPU can load from.  ``PeerBuffers`` builds that table: each rank exports
its own buffer (``h3_ipc_export``: allocation handle + offset), the records
are exchanged with ``torch.distributed.all_gather_object`` over ``group`` (any
backend; gloo needs no GPU), and every peer's buffer is mapped with
``h3_ipc_open``.  The local rank's entry is its own tensor's address.

Ordering is the caller's: the peers' buffers must be written before a rank
call reads them (synchronise, then ``barrier``), and nobody may free or
overwrite a buffer until every rank's kernels reading it have finished
(synchronise, then ``barrier`` again, then ``close``).
"""
from __future__ import annotations

import ctypes as C

import torch
import torch.distributed as dist

from . import _abi


class CudaIpc:
    """The library's CUDA IPC calls (``h3_ipc_export`` / ``_open`` / ``_close``)."""

    def export(self, tensor: torch.Tensor) -> bytes:
        """The tensor's h3_ipc_handle record (allocation handle, offset, size) as bytes."""
        h = _abi.IpcHandle()
        with torch.cuda.device(tensor.device):
            _abi.check(_abi.lib.h3_ipc_export(C.c_void_p(tensor.data_ptr()), C.byref(h)),
                       "h3_ipc_export")
        return bytes(C.string_at(C.addressof(h), C.sizeof(h)))

    @staticmethod
    def _handle(record: bytes) -> _abi.IpcHandle:
        if len(record) != C.sizeof(_abi.IpcHandle):
            raise ValueError("not an h3_ipc_handle record")
        h = _abi.IpcHandle()
        C.memmove(C.addressof(h), record, len(record))
        return h

    def open(self, record: bytes, device: torch.device) -> int:
        """Map a peer's exported buffer on `device`; returns its address there."""
        h = self._handle(record)
        ptr = C.c_void_p()
        with torch.cuda.device(device):
            _abi.check(_abi.lib.h3_ipc_open(C.byref(h), C.byref(ptr)), "h3_ipc_open")
        return int(ptr.value)

    def close(self, address: int, record: bytes, device: torch.device) -> None:
        """Release a mapping made by ``open`` (the last release unmaps it)."""
        h = self._handle(record)
        with torch.cuda.device(device):
            _abi.check(_abi.lib.h3_ipc_close(C.c_void_p(address), C.byref(h)), "h3_ipc_close")


class PeerBuffers:
    """The W ranks' buffers of one kind as addresses usable on this GPU.

    Collective over ``group``: every rank constructs it with its own tensor,
    in the same order as the other ranks' constructions.  ``pointers[r]`` is
    rank r's buffer; ``shapes[r]`` its shape.  ``close()`` unmaps the peers'
    buffers (after the caller's final barrier)."""

    def __init__(self, local: torch.Tensor, group=None, *, ipc=None):
        if not local.is_contiguous():
            raise ValueError("PeerBuffers needs a contiguous tensor")
        self.ipc = ipc if ipc is not None else CudaIpc()
        self.device = local.device
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        record = (self.ipc.export(local), tuple(int(v) for v in local.shape))
        gathered = [None] * self.world
        dist.all_gather_object(gathered, record, group=group)
        self._records = [g[0] for g in gathered]
        self.shapes = [tuple(g[1]) for g in gathered]
        self.pointers = []
        self._opened = []
        try:
            for r in range(self.world):
                if r == self.rank:
                    self.pointers.append(int(local.data_ptr()))
                else:
                    p = self.ipc.open(self._records[r], self.device)
                    self._opened.append((p, self._records[r]))
                    self.pointers.append(p)
        except Exception:
            self.close()
            raise
        self._local = local  # keep the exported buffer alive with the table

    def close(self) -> None:
        """Unmap every peer buffer this table opened (after the caller's final barrier)."""
        while self._opened:
            p, rec = self._opened.pop()
            self.ipc.close(p, rec, self.device)
        self.pointers = []
