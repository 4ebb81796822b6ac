"""Seeded synthetic workloads for the H3 relayout and reduce-scatter path.

This module holds shapes, seeds and random draws only: none of the method's
arithmetic (no partition, no relayout, no reduction).  It is the one module
that both the oracle-side tests and the CUDA-side tests / benchmark import, so
that both see the same input bytes.

Shapes follow H3 as described in "Distributed H3 Execution" (section
"Partition Contract": 56 attention heads of width 128) and the packed QKV /
QKVG operands and 896,000,000-byte window of FastVideo PR #1807 ("Problem and
behavior").  Values are drawn as float32 normals and rounded to BF16 by
torch's round-to-nearest-even cast.  Segment boundaries are distinct uniform
cut points in [1, T-1].  No public dataset exists for this path; all inputs
are synthetic.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

H3_HEADS = 56
H3_HEAD_DIM = 128
H3_HIDDEN = H3_HEADS * H3_HEAD_DIM  # 7168, the projection width used for partials

# Rows generated per randn call, so that the float32 staging buffer stays small
# even for the 14.3 GB long-sequence operand.
_GEN_CHUNK_ELEMS = 1 << 28


@dataclass(frozen=True)
class RelayoutWorkload:
    name: str
    T: int
    P: int
    W: int
    seed: int
    H: int = H3_HEADS
    D: int = H3_HEAD_DIM
    n_segs: int = 1
    seg_lengths: tuple = ()
    window_bytes: int = 0          # 0: one launch over all planes
    inverse_planes: int | None = None  # head->seq operand planes if it differs (attention output)
    description: str = ""

    @property
    def elems(self) -> int:
        return self.T * self.P * self.H * self.D


@dataclass(frozen=True)
class ReduceWorkload:
    name: str
    T: int
    C: int
    W: int
    seed: int
    partial_std: float = 0.5
    bias_std: float = 0.1
    description: str = field(default="")


# The five workloads of the path.  The first is small enough for the full
# oracle; the others are full-size.
TINY_QKV_W2 = RelayoutWorkload(
    "tiny_qkv_T1024_W2", T=1024, P=3, W=2, seed=1, n_segs=3, seg_lengths=(400, 337, 287),
    description="packed QKV BF16 [1024,3,56,128], 3 segments 400/337/287; round trip")
QKV_32K_W6 = RelayoutWorkload(
    "qkv_T32768_W6", T=32768, P=3, W=6, seed=2, n_segs=8,
    description="packed QKV BF16 [32768,3,56,128], ragged heads 10,10,9,9,9,9, 8 random segments; both directions")
QKVG_128K_W4 = RelayoutWorkload(
    "qkvg_T131072_W4", T=131072, P=4, W=4, seed=3, n_segs=16, inverse_planes=1,
    description="packed QKVG BF16 [131072,4,56,128] seq->head; attention output [131072,56,128] head->seq")
RS_64K_W8 = ReduceWorkload(
    "reduce_scatter_T65536_C7168_W8", T=65536, C=H3_HIDDEN, W=8, seed=4,
    description="8 BF16 partials [65536,7168] N(0,0.5), bias [7168] N(0,0.1)")
QKVG_250K_W4_CHUNKED = RelayoutWorkload(
    "qkvg_T250000_W4_chunked", T=250000, P=4, W=4, seed=5, n_segs=1, window_bytes=896_000_000,
    description="packed QKVG BF16 [250000,4,56,128], one plane per launch under an 896,000,000-byte window; both directions")

# The long sequence over two ranks: one plane of one rank (1,792,000,000 bytes)
# is twice the window, so each plane moves in token chunks.
QKVG_250K_W2_CHUNKED = RelayoutWorkload(
    "qkvg_T250000_W2_chunked", T=250000, P=4, W=2, seed=6, n_segs=1, window_bytes=896_000_000,
    description="packed QKVG BF16 [250000,4,56,128] over 2 ranks; planes larger than the window, two token chunks each")

WORKLOADS = {w.name: w for w in (TINY_QKV_W2, QKV_32K_W6, QKVG_128K_W4, RS_64K_W8,
                                 QKVG_250K_W4_CHUNKED, QKVG_250K_W2_CHUNKED)}


def _generator(seed: int, device) -> torch.Generator:
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    return g


def normal_bf16(shape, seed: int, std: float = 1.0, device="cpu") -> torch.Tensor:
    """BF16 tensor of N(0, std^2) draws (std is a standard deviation)."""
    shape = tuple(int(s) for s in shape)
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    g = _generator(seed, device)
    n = flat.numel()
    for lo in range(0, n, _GEN_CHUNK_ELEMS):
        hi = min(n, lo + _GEN_CHUNK_ELEMS)
        x = torch.randn(hi - lo, generator=g, dtype=torch.float32, device=device)
        if std != 1.0:
            x.mul_(std)
        flat[lo:hi].copy_(x)
        del x
    return out


def packed_operand(w: RelayoutWorkload, planes: int | None = None, device="cpu",
                   seed_offset: int = 0) -> torch.Tensor:
    """Packed sequence operand [T, P, H, D] BF16 ~ N(0,1)."""
    P = w.P if planes is None else planes
    return normal_bf16((w.T, P, w.H, w.D), w.seed + seed_offset, 1.0, device)


def segment_bounds(T: int, n_segs: int, seed: int, lengths=()) -> np.ndarray:
    """Packed segment boundaries b_0=0 < b_1 < ... < b_n = T (int64).

    With explicit lengths they are used as given; otherwise n_segs-1 distinct
    cut points are drawn uniformly from [1, T-1] and sorted."""
    if lengths:
        b = np.concatenate([[0], np.cumsum(np.asarray(lengths, dtype=np.int64))])
        assert b[-1] == T, "segment lengths must add up to T"
        return b.astype(np.int64)
    if n_segs <= 1:
        return np.array([0, T], dtype=np.int64)
    rng = np.random.default_rng(seed)
    cuts = np.sort(rng.choice(np.arange(1, T, dtype=np.int64), size=n_segs - 1, replace=False))
    return np.concatenate([[0], cuts, [T]]).astype(np.int64)


def partials_and_bias(w: ReduceWorkload, device="cpu"):
    """W partials BF16 [W, T, C] ~ N(0, partial_std^2) and bias BF16 [C] ~ N(0, bias_std^2)."""
    partials = normal_bf16((w.W, w.T, w.C), w.seed, w.partial_std, device)
    bias = normal_bf16((w.C,), w.seed + 1_000_003, w.bias_std, device)
    return partials, bias


def index_coded(shape, device="cpu") -> torch.Tensor:
    """BF16-typed tensor whose 16-bit patterns are the flat element index mod 2^16.

    For tensors of at most 65,536 elements every element carries a distinct
    pattern, so any misplaced element is visible."""
    n = int(np.prod(shape))
    codes = (torch.arange(n, dtype=torch.int64) & 0xFFFF).to(torch.int32)
    codes = torch.where(codes >= 0x8000, codes - 0x10000, codes).to(torch.int16)
    return codes.view(torch.bfloat16).reshape(shape).to(device)


def random_bits(shape, seed: int, device="cpu") -> torch.Tensor:
    """BF16-typed tensor of uniformly random 16-bit patterns (NaN/Inf included)."""
    g = torch.Generator().manual_seed(seed)
    bits = torch.randint(-32768, 32768, tuple(shape), generator=g, dtype=torch.int32)
    return bits.to(torch.int16).view(torch.bfloat16).to(device)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw 16-bit patterns of a BF16 tensor as a host numpy uint16 array."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
