"""Helpers for the GPU parity tests: host copies of BF16 bit patterns, guard
bands around outputs, and sampled oracle checks at full sizes."""
from __future__ import annotations

import numpy as np
import torch

import workloads as wl

GUARD_ELEMS = 4096  # canary elements on each side of a guarded output
CANARY = 0x5A5A


def bits(t: torch.Tensor) -> np.ndarray:
    return wl.bf16_bits(t)


def guarded(shape, device, dtype=torch.bfloat16):
    """An output tensor with canary bands before and after it in one allocation."""
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * GUARD_ELEMS,), CANARY, dtype=torch.int16, device=device)
    # keep the interior 16-byte aligned: GUARD_ELEMS * 2 bytes is a multiple of 16
    out = buf[GUARD_ELEMS:GUARD_ELEMS + n].view(dtype).view(shape)
    return buf, out


def guards_intact(buf: torch.Tensor) -> bool:
    head = buf[:GUARD_ELEMS]
    tail = buf[-GUARD_ELEMS:]
    return bool((head == CANARY).all().item() and (tail == CANARY).all().item())


def _flat16(t: torch.Tensor) -> torch.Tensor:
    return t.reshape(-1).view(torch.int16)


def edge_indices(T, P, Hj, D, token_starts) -> np.ndarray:
    """Flat indices of a [T, P, Hj, D] buffer at rank token boundaries and head edges."""
    toks = sorted({0, T - 1} | {int(s) for s in token_starts[1:-1]} |
                  {int(s) - 1 for s in token_starts[1:-1]})
    idx = []
    for t in toks:
        for p in {0, P - 1}:
            for h in {0, Hj - 1}:
                for d in {0, D - 1}:
                    idx.append(((t * P + p) * Hj + h) * D + d)
    return np.array(sorted(set(idx)), dtype=np.int64)


def sampled_check_seq_to_head(o, send, recv, T, P, H, D, W, n=200_000, seed=0):
    """Compare sampled elements of every head-side output with the oracle's
    gather map applied to the sequence-side inputs."""
    rng = np.random.default_rng(seed)
    dev = recv[0].device
    ts = o.partition_range(T, W)
    hs = o.partition_range(H, W)
    src_flat = [_flat16(s) for s in send]
    for j in range(W):
        Hj = int(hs[j + 1] - hs[j])
        out = _flat16(recv[j])
        idx = np.concatenate([rng.integers(0, out.numel(), size=n, dtype=np.int64),
                              edge_indices(T, P, Hj, D, ts)])
        src_rank, src_elem = o.seq_to_head_locate(T, P, H, D, W, j, idx)
        got = out[torch.from_numpy(idx).to(dev)].cpu().numpy()
        want = np.empty_like(got)
        for r in range(W):
            m = src_rank == r
            if m.any():
                want[m] = src_flat[r][torch.from_numpy(src_elem[m]).to(dev)].cpu().numpy()
        bad = np.flatnonzero(got != want)
        assert bad.size == 0, f"rank {j}: {bad.size} mismatches, first at element {idx[bad[0]]}"


def sampled_check_head_to_seq(o, send, recv, T, P, H, D, W, n=200_000, seed=0):
    """Compare sampled elements of every sequence-side output with the oracle's
    gather map applied to the head-side inputs."""
    rng = np.random.default_rng(seed)
    dev = recv[0].device
    ts = o.partition_range(T, W)
    src_flat = [_flat16(s) for s in send]
    for r in range(W):
        Tr = int(ts[r + 1] - ts[r])
        out = _flat16(recv[r])
        idx = np.concatenate([rng.integers(0, out.numel(), size=n, dtype=np.int64),
                              edge_indices(Tr, P, H, D, [0, Tr])])
        src_rank, src_elem = o.head_to_seq_locate(T, P, H, D, W, r, idx)
        got = out[torch.from_numpy(idx).to(dev)].cpu().numpy()
        want = np.empty_like(got)
        for j in range(W):
            m = src_rank == j
            if m.any():
                want[m] = src_flat[j][torch.from_numpy(src_elem[m]).to(dev)].cpu().numpy()
        bad = np.flatnonzero(got != want)
        assert bad.size == 0, f"rank {r}: {bad.size} mismatches, first at element {idx[bad[0]]}"


def same_bits(a: torch.Tensor, b: torch.Tensor) -> bool:
    return a.shape == b.shape and torch.equal(a.contiguous().view(torch.int16),
                                              b.contiguous().view(torch.int16))


def nan_aware_equal(got: np.ndarray, want: np.ndarray) -> np.ndarray:
    """Element mask of agreement: equal patterns, or both NaN (any NaN)."""
    def is_nan(x):
        return ((x & 0x7F80) == 0x7F80) & ((x & 0x7F) != 0)
    return (got == want) | (is_nan(got) & is_nan(want))


def chunk_window(kind, T, H, D, W):
    """Window bytes for a chunked-mode test: 0 (unchunked), "plane" (exactly
    one plane of the largest rank, one launch per plane), "sub" (half of that,
    so every plane is split into token chunks) or "min" (one token of every
    rank: one-token chunks)."""
    if not kind:
        return 0
    tmax, hmax = -(-T // W), -(-H // W)
    row, head = H * D * 2, D * 2
    smallest = max(row, W * hmax * head)
    plane = max(tmax * row, T * hmax * head)
    return {"plane": plane, "sub": max(smallest, plane // 2), "min": smallest}[kind]


def range_window(kind, T, P, H, D, W):
    """Window bytes for token ranges over all planes (H3_LAUNCH_CHUNK_TOKENS):
    "plane" (one plane of the largest rank: about P ranges), "half" (half of
    that) or "min" (one token of every plane of every rank: one-token
    ranges)."""
    tmax, hmax = -(-T // W), -(-H // W)
    row, head = H * D * 2, D * 2
    smallest = P * max(row, W * hmax * head)
    plane = max(tmax * row, T * hmax * head)
    return {"plane": max(smallest, plane), "half": max(smallest, plane // 2), "min": smallest}[kind]
