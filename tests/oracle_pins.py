"""Pins of the CPU oracle to facts outside the oracle itself.

Each ``check_*`` takes an ``oracle.Oracle`` and raises ``AssertionError`` when
the oracle disagrees with what the pages or the mathematics fix:

* the head table printed in "Distributed H3 Execution", section "Partition
  Contract" (tests/golden/head_partition_table.txt);
* hand-derived segment clip cases and invariants (same section);
* relayouts against numpy slicing of index-coded tensors (every element of a
  tiny tensor carries a distinct 16-bit pattern), the world-size-one identity
  ("Distributed H3 Execution", section "Validation": one-rank runs) and the
  sequence->head->sequence round trip ("Ulysses transport identity at 2, 4, 6
  and 8 ranks", same section);
* BF16 rounding against hand-derived IEEE cases and torch's CPU cast;
* the reduce-scatter against hand-derived single-element cases
  (tests/golden/reduce_order_cases.txt), an integer split-GEMM whose sharded
  partials must add up to the unsharded product with the bias once, and a
  row-assignment probe.

The module is also run against deliberately broken copies of the oracle
(tests/test_oracle_mutants.py): every planted mistake must fail at least one
check here.
"""
from __future__ import annotations

import json
import os
import struct

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# --------------------------------------------------------------------------
# helpers (no method arithmetic)
# --------------------------------------------------------------------------

def _f32_bits(x: float) -> int:
    return struct.unpack("<I", struct.pack("<f", x))[0]


def _bf16_bits_of_exact(x: float) -> int:
    """Bit pattern of a value that is exactly representable in BF16."""
    u = _f32_bits(x)
    assert (u & 0xFFFF) == 0, f"{x!r} is not exactly representable in BF16"
    return u >> 16


def _parse_value(s: str) -> float:
    s = s.strip()
    if s == "-0":
        return -0.0
    if s in ("inf", "-inf", "nan"):
        return float(s)
    if "0x" in s:
        return float.fromhex(s)
    return float(s)


def _is_nan_bf16(b: int) -> bool:
    return (b & 0x7F80) == 0x7F80 and (b & 0x7F) != 0


def _index_coded(shape) -> np.ndarray:
    n = int(np.prod(shape))
    assert n <= 65536
    return np.arange(n, dtype=np.uint16).reshape(shape)


def _golden_head_table():
    table = {}
    with open(os.path.join(GOLDEN, "head_partition_table.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            w, sizes = line.split(":")
            table[int(w)] = [int(v) for v in sizes.split()]
    return table


# --------------------------------------------------------------------------
# partition contract
# --------------------------------------------------------------------------

def check_head_table(o):
    table = _golden_head_table()
    assert sorted(table) == [2, 4, 6, 8]
    for w, sizes in table.items():
        starts = o.partition_range(56, w)
        assert list(np.diff(starts)) == sizes, (w, list(np.diff(starts)), sizes)


def check_partition_invariants(o):
    rng = np.random.default_rng(11)
    cases = [(1, 1), (56, 1), (56, 56), (1000, 6), (32768, 6), (250000, 4), (7, 3)]
    cases += [(int(rng.integers(1, 5000)), int(rng.integers(1, 64))) for _ in range(200)]
    for n, w in cases:
        if n < w:
            continue
        s = o.partition_range(n, w)
        sizes = np.diff(s)
        assert s[0] == 0 and s[-1] == n, (n, w)
        assert sizes.min() >= 1
        assert sizes.max() - sizes.min() <= 1, (n, w, sizes)
        # the remainder goes to the first ranks (W=6 row of the head table)
        assert all(sizes[i] >= sizes[i + 1] for i in range(w - 1)), (n, w, sizes)
    assert list(o.partition_range(1234, 1)) == [0, 1234]
    for n, w in [(3, 4), (0, 1), (5, 0), (55, 56)]:
        try:
            o.partition_range(n, w)
        except ValueError:
            continue
        raise AssertionError(f"empty partition accepted: n={n} w={w}")
    # owner lookup agrees with the ranges
    s = o.partition_range(1000, 6)
    for x in [0, 166, 167, 333, 334, 999]:
        r = o.owner(s, x)
        assert s[r] <= x < s[r + 1], (x, r)


def check_segment_clip_golden(o):
    with open(os.path.join(GOLDEN, "segment_clip_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        s = o.partition_range(c["T"], c["W"])
        assert list(s) == c["token_starts"], (c["note"], list(s))
        for r, want in enumerate(c["ranks"]):
            lb, ids = o.clip_segments(c["bounds"], int(s[r]), int(s[r + 1]))
            assert list(lb) == want["local_bounds"], (c["note"], r, list(lb))
            assert list(ids) == want["seg_ids"], (c["note"], r, list(ids))


def check_segment_clip_invariants(o):
    rng = np.random.default_rng(12)
    for _ in range(100):
        T = int(rng.integers(1, 400))
        W = int(rng.integers(1, min(T, 9) + 1))
        S = int(rng.integers(1, min(T, 12) + 1))
        cuts = np.sort(rng.choice(np.arange(1, T), size=S - 1, replace=False)) if S > 1 else []
        bounds = np.concatenate([[0], cuts, [T]]).astype(np.int64)
        s = o.partition_range(T, W)
        covered = np.zeros(S, dtype=np.int64)
        for r in range(W):
            lb, ids = o.clip_segments(bounds, int(s[r]), int(s[r + 1]))
            assert lb[0] == 0 and lb[-1] == s[r + 1] - s[r]
            assert np.all(np.diff(lb) > 0)
            assert np.all(np.diff(ids) == 1) if len(ids) > 1 else True
            for k, a, b in zip(ids, lb[:-1], lb[1:]):
                ga, gb = a + s[r], b + s[r]
                assert bounds[k] <= ga < gb <= bounds[k + 1]
                covered[k] += gb - ga
        assert np.array_equal(covered, np.diff(bounds))
        if W == 1:
            lb, ids = o.clip_segments(bounds, 0, T)
            assert np.array_equal(lb, bounds) and list(ids) == list(range(S))


# --------------------------------------------------------------------------
# relayouts
# --------------------------------------------------------------------------

_RELAYOUT_SHAPES = [
    # T, P, H, D, W
    (8, 3, 56, 2, 2),
    (10, 3, 56, 1, 6),
    (9, 4, 56, 1, 8),
    (12, 3, 56, 4, 4),
    (7, 3, 5, 4, 3),
    (5, 1, 5, 3, 5),
    (13, 2, 9, 8, 1),
    (6, 2, 7, 16, 4),
]


def _split_rows(full: np.ndarray, starts: np.ndarray):
    return [full[starts[r]:starts[r + 1]] for r in range(len(starts) - 1)]


def check_relayout_slicing(o):
    for T, P, H, D, W in _RELAYOUT_SHAPES:
        full = _index_coded((T, P, H, D))
        ts = o.partition_range(T, W)
        hs = o.partition_range(H, W)
        send = _split_rows(full, ts)
        recv = o.seq_to_head(send, T, P, H, D, W)
        for j in range(W):
            want = full[:, :, hs[j]:hs[j + 1], :]
            assert recv[j].shape == want.shape
            assert np.array_equal(recv[j], want), ("seq->head", T, P, H, D, W, j)
        # head -> seq on an independent index-coded head-side operand
        heads = [(_index_coded((T, P, hs[j + 1] - hs[j], D)) + np.uint16(17 * j)) for j in range(W)]
        back = o.head_to_seq(heads, T, P, H, D, W)
        joined = np.concatenate(heads, axis=2)
        for r in range(W):
            want = joined[ts[r]:ts[r + 1]]
            assert np.array_equal(back[r], want), ("head->seq", T, P, H, D, W, r)


def check_world_one_identity(o):
    x = _index_coded((11, 3, 7, 8))
    (y,) = o.seq_to_head([x], 11, 3, 7, 8, 1)
    assert np.array_equal(y, x)
    (z,) = o.head_to_seq([x], 11, 3, 7, 8, 1)
    assert np.array_equal(z, x)


def check_round_trip(o):
    rng = np.random.default_rng(13)
    for W in (2, 4, 6, 8):
        for T in (W, 50, 97):
            P, H, D = 3, 56, 8
            full = rng.integers(0, 1 << 16, size=(T, P, H, D), dtype=np.uint16)
            ts = o.partition_range(T, W)
            send = _split_rows(full, ts)
            back = o.head_to_seq(o.seq_to_head(send, T, P, H, D, W), T, P, H, D, W)
            for r in range(W):
                assert np.array_equal(back[r], send[r]), (W, T, r)


def check_locate_matches_full(o):
    for T, P, H, D, W in _RELAYOUT_SHAPES[:5]:
        full = _index_coded((T, P, H, D))
        ts = o.partition_range(T, W)
        send = _split_rows(full, ts)
        recv = o.seq_to_head(send, T, P, H, D, W)
        for j in range(W):
            idx = np.arange(recv[j].size, dtype=np.int64)
            src_rank, src_elem = o.seq_to_head_locate(T, P, H, D, W, j, idx)
            got = np.array([send[r].reshape(-1)[e] for r, e in zip(src_rank, src_elem)],
                           dtype=np.uint16)
            assert np.array_equal(got, recv[j].reshape(-1)), ("locate s2h", j)
        back = o.head_to_seq(recv, T, P, H, D, W)
        for r in range(W):
            idx = np.arange(back[r].size, dtype=np.int64)
            src_rank, src_elem = o.head_to_seq_locate(T, P, H, D, W, r, idx)
            got = np.array([recv[j].reshape(-1)[e] for j, e in zip(src_rank, src_elem)],
                           dtype=np.uint16)
            assert np.array_equal(got, back[r].reshape(-1)), ("locate h2s", r)


# --------------------------------------------------------------------------
# BF16 rounding
# --------------------------------------------------------------------------

def check_bf16_golden(o):
    n = 0
    with open(os.path.join(GOLDEN, "bf16_rne_cases.txt")) as f:
        for line in f:
            body = line.split("#", 1)[0].strip()
            if not body:
                continue
            src_hex, want = body.split()
            # build the binary32 input from its bits: a Python float would
            # quieten a signalling NaN on the way in
            xa = np.array([int(src_hex, 16)], dtype=np.uint32).view(np.float32)
            got = int(o.f32_to_bf16(xa)[0])
            x = float(xa[0])
            single = int(o.lib.h3o_f32_to_bf16_rne(x)) if not np.isnan(x) else got
            assert got == single
            if want == "nan":
                assert _is_nan_bf16(got), (src_hex, hex(got))
            else:
                assert got == int(want, 16), (src_hex, hex(got), want)
            n += 1
    assert n >= 20


def check_bf16_vs_torch(o):
    g = torch.Generator().manual_seed(14)
    bits = torch.randint(-(1 << 31), 1 << 31, (1 << 18,), generator=g, dtype=torch.int64)
    x = bits.to(torch.int32).view(torch.float32)
    x = torch.cat([x, torch.randn(1 << 18, generator=g) * 3.0,
                   torch.randn(1 << 12, generator=g) * 1e-39])
    x = x[~torch.isnan(x)]
    want = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = o.f32_to_bf16(x.numpy())
    assert np.array_equal(got, want), int(np.count_nonzero(got != want))
    # widening is exact: agrees with torch's BF16 -> float32
    b = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16)
    wide = b.view(torch.bfloat16).float().numpy()
    mine = o.bf16_to_f32(b.numpy().view(np.uint16))
    assert np.array_equal(wide.view(np.uint32), mine.view(np.uint32))


# --------------------------------------------------------------------------
# reduce-scatter
# --------------------------------------------------------------------------

def _reduce_cases():
    cases = []
    with open(os.path.join(GOLDEN, "reduce_order_cases.txt")) as f:
        for line in f:
            body = line.split("#", 1)[0].strip()
            if not body:
                continue
            parts, bias, want = (s.strip() for s in body.split("|"))
            vals = [_parse_value(v) for v in parts.split(",")]
            b = None if bias == "none" else _parse_value(bias)
            cases.append((vals, b, _parse_value(want), line.strip()))
    return cases


def check_reduce_golden(o):
    cases = _reduce_cases()
    assert len(cases) >= 12
    for vals, b, want, line in cases:
        W = len(vals)
        partials = [np.array([[_bf16_bits_of_exact(v)]], dtype=np.uint16) for v in vals]
        bias = None if b is None else np.array([_bf16_bits_of_exact(b)], dtype=np.uint16)
        got = int(o.reduce_rows(partials, bias)[0, 0])
        if np.isnan(want):
            assert _is_nan_bf16(got), (line, hex(got))
        else:
            assert got == _bf16_bits_of_exact(want), (line, hex(got))
        # the same element through the full scatter (every row carries the case)
        rows = [np.full((W, 3), p[0, 0], dtype=np.uint16) for p in partials]
        b3 = None if bias is None else np.full(3, bias[0], dtype=np.uint16)
        outs = o.ragged_reduce_scatter(rows, b3, W)
        for out in outs:
            if np.isnan(want):
                assert all(_is_nan_bf16(int(v)) for v in out.reshape(-1)), line
            else:
                assert np.all(out == _bf16_bits_of_exact(want)), line


def check_split_gemm(o):
    """Sharded partials of an integer GEMM add up to the unsharded product + bias once."""
    rng = np.random.default_rng(15)
    for T, K, Cc, W in [(12, 12, 16, 3), (40, 12, 8, 6), (9, 8, 24, 8), (5, 4, 8, 1)]:
        X = rng.integers(-4, 5, size=(T, K)).astype(np.int64)
        Wt = rng.integers(-4, 5, size=(Cc, K)).astype(np.int64)
        b = rng.integers(-8, 9, size=Cc).astype(np.int64)
        ks = o.partition_range(K, W) if K >= W else None
        if ks is None:
            continue
        partials = []
        for w in range(W):
            part = X[:, ks[w]:ks[w + 1]] @ Wt[:, ks[w]:ks[w + 1]].T
            assert np.abs(part).max() <= 256
            partials.append(np.array([[_bf16_bits_of_exact(float(v)) for v in row] for row in part],
                                     dtype=np.uint16))
        bias = np.array([_bf16_bits_of_exact(float(v)) for v in b], dtype=np.uint16)
        full = X @ Wt.T + b[None, :]
        assert np.abs(full).max() <= 256
        outs = o.ragged_reduce_scatter(partials, bias, W)
        ts = o.partition_range(T, W)
        for r in range(W):
            want = np.array([[_bf16_bits_of_exact(float(v)) for v in row]
                             for row in full[ts[r]:ts[r + 1]]], dtype=np.uint16)
            assert np.array_equal(outs[r], want), (T, K, Cc, W, r)


def check_reduce_row_assignment(o):
    """Rank r receives rows ts_r..te_r-1: partial 0 carries the row number."""
    for T, W in [(200, 6), (97, 8), (9, 2), (5, 5)]:
        Cc = 8
        p0 = np.array([[_bf16_bits_of_exact(float(t))] * Cc for t in range(T)], dtype=np.uint16)
        zeros = [np.zeros((T, Cc), dtype=np.uint16) for _ in range(W - 1)]
        outs = o.ragged_reduce_scatter([p0] + zeros, None, W)
        sizes = [T // W + (1 if r < T % W else 0) for r in range(W)]
        t = 0
        for r in range(W):
            assert outs[r].shape == (sizes[r], Cc)
            for tl in range(sizes[r]):
                assert np.all(outs[r][tl] == _bf16_bits_of_exact(float(t))), (T, W, r, tl)
                t += 1


def check_reduce_identities(o):
    rng = np.random.default_rng(16)
    T, Cc = 33, 40
    bias = o.f32_to_bf16(rng.normal(0, 0.1, Cc).astype(np.float32))
    bias[bias == 0x8000] = 0x3F80  # keep -0 out: +0 + -0 is +0
    zeros = [np.zeros((T, Cc), dtype=np.uint16) for _ in range(5)]
    for out in o.ragged_reduce_scatter(zeros, bias, 5):
        assert np.all(out == bias[None, :])
    # one rank, no bias: the output is the input (finite values)
    x = o.f32_to_bf16(rng.normal(0, 1, (T, Cc)).astype(np.float32))
    (y,) = o.ragged_reduce_scatter([x], None, 1)
    assert np.array_equal(x, y)
    # sum with exact zeros elsewhere returns the non-zero partial
    outs = o.ragged_reduce_scatter([zeros[0], x, zeros[1]], None, 3)
    assert np.array_equal(np.concatenate(outs), x)


def check_all_gather(o):
    """Every rank holds all rows: numpy concatenation of the rank blocks,
    row-number coded rows, W=1 identity, and reduce-scatter followed by
    all-gather reproducing the unsharded integer GEMM plus bias."""
    rng = np.random.default_rng(17)
    for T, Cc, W in [(10, 8, 3), (97, 16, 8), (5, 8, 5), (33, 24, 1), (64, 8, 6)]:
        full = rng.integers(0, 1 << 16, size=(T, Cc), dtype=np.uint16)
        ts = o.partition_range(T, W)
        blocks = [full[ts[r]:ts[r + 1]] for r in range(W)]
        outs = o.ragged_all_gather(blocks, W)
        for j in range(W):
            assert np.array_equal(outs[j], np.concatenate(blocks, axis=0)), (T, W, j)
        coded = [np.array([[_bf16_bits_of_exact(float(t))] * Cc for t in range(ts[r], ts[r + 1])],
                          dtype=np.uint16).reshape(-1, Cc) for r in range(W)]
        for out in o.ragged_all_gather(coded, W):
            for t in range(T):
                assert np.all(out[t] == _bf16_bits_of_exact(float(t)))
    # reduce-scatter then all-gather: every rank ends with X W^T + b
    T, K, Cc, W = 40, 12, 8, 6
    X = rng.integers(-4, 5, size=(T, K))
    Wt = rng.integers(-4, 5, size=(Cc, K))
    b = rng.integers(-8, 9, size=Cc)
    ks = o.partition_range(K, W)
    partials = [np.array([[_bf16_bits_of_exact(float(v)) for v in row]
                          for row in X[:, ks[w]:ks[w + 1]] @ Wt[:, ks[w]:ks[w + 1]].T], dtype=np.uint16)
                for w in range(W)]
    bias = np.array([_bf16_bits_of_exact(float(v)) for v in b], dtype=np.uint16)
    gathered = o.ragged_all_gather(o.ragged_reduce_scatter(partials, bias, W), W)
    want = np.array([[_bf16_bits_of_exact(float(v)) for v in row] for row in X @ Wt.T + b[None, :]],
                    dtype=np.uint16)
    for g in gathered:
        assert np.array_equal(g, want)


def check_plane_major_layouts(o):
    """Plane-major buffers are numpy transposes of the token-major ones: for
    every layout pair the relayout equals the token-major result with the
    (token, plane) axes swapped where a side is plane-major; round trips are
    the identity."""
    for T, P, H, D, W in [(10, 3, 56, 1, 6), (7, 3, 5, 4, 3), (9, 4, 56, 1, 8), (13, 2, 9, 8, 1)]:
        full = _index_coded((T, P, H, D))
        ts = o.partition_range(T, W)
        send_tm = _split_rows(full, ts)
        ref = o.seq_to_head(send_tm, T, P, H, D, W)          # token-major both sides
        for spm in (False, True):
            for hpm in (False, True):
                send = [np.ascontiguousarray(x.transpose(1, 0, 2, 3)) if spm else x for x in send_tm]
                got = o.relayout_layout(send, T, P, H, D, W, True, spm, hpm)
                for j in range(W):
                    want = np.ascontiguousarray(ref[j].transpose(1, 0, 2, 3)) if hpm else ref[j]
                    assert np.array_equal(got[j], want), ("s2h", spm, hpm, j)
                back = o.relayout_layout(got, T, P, H, D, W, False, spm, hpm)
                for r in range(W):
                    assert np.array_equal(back[r], send[r]), ("h2s", spm, hpm, r)


def _bf16_of(x: np.ndarray) -> np.ndarray:
    """BF16 patterns of float32 values by torch's CPU round-to-nearest-even cast."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _f32_of(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32)


def check_gated_reduce_scatter(o):
    """Fused reduce-scatter + gating equals the reduce-scatter followed by
    the gating written with numpy binary32 arithmetic and torch's BF16 cast;
    gate 0 leaves x; gate 1 on x = 0 gives the reduce-scatter; per-segment
    gate values k+1 show each row's segment, matching the clip cases."""
    rng = np.random.default_rng(18)
    for T, Cc, W, bounds in [(10, 8, 3, [0, 2, 9, 10]), (1024, 16, 2, [0, 400, 737, 1024]),
                             (97, 8, 8, [0, 5, 6, 50, 97]), (9, 8, 3, [0, 3, 6, 9]), (33, 24, 1, [0, 33])]:
        S = len(bounds) - 1
        partials = [o.f32_to_bf16(rng.normal(0, 0.5, (T, Cc)).astype(np.float32)) for _ in range(W)]
        bias = o.f32_to_bf16(rng.normal(0, 0.1, Cc).astype(np.float32))
        gate = o.f32_to_bf16(rng.normal(0, 1.0, (S, Cc)).astype(np.float32))
        ts = o.partition_range(T, W)
        x = [o.f32_to_bf16(rng.normal(0, 1.0, (ts[r + 1] - ts[r], Cc)).astype(np.float32)) for r in range(W)]
        got = o.reduce_scatter_gated(partials, bias, gate, bounds, x, W)
        y = o.ragged_reduce_scatter(partials, bias, W)
        seg = np.searchsorted(np.asarray(bounds), np.arange(T), side="right") - 1
        for r in range(W):
            rows = np.arange(ts[r], ts[r + 1])
            want = _bf16_of(_f32_of(x[r]) + _f32_of(gate[seg[rows]]) * _f32_of(y[r]))
            assert np.array_equal(got[r], want), (T, W, r)
        zero = [np.zeros(S * Cc, np.uint16).reshape(S, Cc)][0]
        got0 = o.reduce_scatter_gated(partials, bias, zero, bounds, x, W)
        for r in range(W):
            # x + (+-0) is x, except that -0 + +0 is +0: compare where x is not -0
            keep = x[r] != 0x8000
            assert np.array_equal(got0[r][keep], x[r][keep])
        one = np.full((S, Cc), 0x3F80, np.uint16)
        xz = [np.zeros_like(v) for v in x]
        got1 = o.reduce_scatter_gated(partials, bias, one, bounds, xz, W)
        for r in range(W):
            # +0 + y is y except that y = -0 gives +0
            assert np.array_equal(got1[r], np.where(y[r] == 0x8000, 0, y[r]).astype(np.uint16))
    # segment of each row through the clip: gate row k holds k+1, y = 1
    with open(os.path.join(GOLDEN, "segment_clip_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        T, W, bounds = c["T"], c["W"], c["bounds"]
        S = len(bounds) - 1
        Cc = 8
        partials = [np.full((T, Cc), 0x3F80 if w == 0 else 0, np.uint16) for w in range(W)]
        gate = np.array([[_bf16_bits_of_exact(float(k + 1))] * Cc for k in range(S)], np.uint16)
        ts = o.partition_range(T, W)
        x = [np.zeros((ts[r + 1] - ts[r], Cc), np.uint16) for r in range(W)]
        got = o.reduce_scatter_gated(partials, None, gate, bounds, x, W)
        for r, want in enumerate(c["ranks"]):
            lb, ids = want["local_bounds"], want["seg_ids"]
            for k, a, b in zip(ids, lb[:-1], lb[1:]):
                assert np.all(got[r][a:b] == _bf16_bits_of_exact(float(k + 1))), (c["note"], r, k)


ALL_CHECKS = [
    check_head_table,
    check_partition_invariants,
    check_segment_clip_golden,
    check_segment_clip_invariants,
    check_relayout_slicing,
    check_world_one_identity,
    check_round_trip,
    check_locate_matches_full,
    check_bf16_golden,
    check_bf16_vs_torch,
    check_reduce_golden,
    check_split_gemm,
    check_reduce_row_assignment,
    check_reduce_identities,
    check_all_gather,
    check_plane_major_layouts,
    check_gated_reduce_scatter,
]


def run_all(o) -> list[str]:
    """Run every check; return the names of those that failed."""
    failed = []
    for chk in ALL_CHECKS:
        try:
            chk(o)
        except AssertionError:
            failed.append(chk.__name__)
        except ValueError:
            failed.append(chk.__name__)
    return failed
