"""Property-based checks of the host plan (h3_partition) against the oracle,
over shapes hypothesis chooses: token and head ranges equal the oracle's
quotient/remainder split, and every rank's clipped, rebased segment pieces
equal the oracle's clip; the pieces of each segment tile it exactly."""
import numpy as np
from hypothesis import given, settings, strategies as st

import ragged_reduce_b200 as rr


@st.composite
def plans(draw):
    W = draw(st.integers(1, 64))
    T = draw(st.integers(W, 5_000_000))
    H = draw(st.integers(W, 256))
    S = draw(st.integers(1, min(T, 48)))
    cuts = draw(st.lists(st.integers(1, T - 1), min_size=S - 1, max_size=S - 1, unique=True)) \
        if T > 1 and S > 1 else []
    bounds = np.array([0] + sorted(cuts) + [T], dtype=np.int64)
    return T, H, W, bounds


@settings(max_examples=300, deadline=None, derandomize=True)
@given(plans())
def test_partition_agrees_with_the_oracle(oracle_lib, plan):
    T, H, W, bounds = plan
    p = rr.partition(T, H, W, bounds)
    assert np.array_equal(p.token_starts, oracle_lib.partition_range(T, W))
    assert np.array_equal(p.head_starts.astype(np.int64), oracle_lib.partition_range(H, W))
    covered = np.zeros(len(bounds) - 1, dtype=np.int64)
    for r in range(W):
        ts, te = int(p.token_starts[r]), int(p.token_starts[r + 1])
        lb, ids = oracle_lib.clip_segments(bounds, ts, te)
        assert np.array_equal(p.local_bounds[r], lb)
        assert np.array_equal(p.seg_ids[r], ids)
        assert lb[0] == 0 and lb[-1] == te - ts and np.all(np.diff(lb) > 0)
        np.add.at(covered, ids, np.diff(lb))
    assert np.array_equal(covered, np.diff(bounds))
