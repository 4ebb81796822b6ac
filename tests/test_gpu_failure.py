"""Failure handling on the GPU without a fault: the bulk kernels' bounded
barrier wait gives up, reports it, and the context stays usable.

``h3_bounded_wait_selftest`` waits on a shared-memory barrier that nothing
arrives at (the "flag that nothing sets"); the wait must expire after its
poll limit and report it.  A barrier completed first must not expire.  Then
ordinary calls still run and match the oracle."""
import time

import numpy as np
import pytest

import ragged_reduce_b200 as rr
import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.mark.parametrize("polls", [1, 64, 4096])
def test_wait_on_a_barrier_nothing_completes_expires(polls):
    t0 = time.perf_counter()
    assert rr.bounded_wait_selftest(polls, arrive_first=False) is True
    elapsed = time.perf_counter() - t0
    assert elapsed < 30.0, f"{polls} polls took {elapsed:.2f} s"


@pytest.mark.parametrize("polls", [1, 64])
def test_wait_on_a_completed_barrier_succeeds(polls):
    assert rr.bounded_wait_selftest(polls, arrive_first=True) is False


def test_context_usable_after_an_expired_wait(oracle_lib):
    assert rr.bounded_wait_selftest(16, arrive_first=False) is True
    T, P, H, D, W = 600, 3, 56, 128, 4
    part = rr.partition(T, H, W)
    x = wl.random_bits((T, P, H, D), 91, DEV)
    send = rr.split_rows(x, part.token_starts)
    heads = rr.alloc_head_side(T, P, H, D, W, DEV)
    rr.seq_to_head(send, heads, variant=rr.H3_VARIANT_BULK)
    want = oracle_lib.seq_to_head([gu.bits(s) for s in send], T, P, H, D, W)
    for j in range(W):
        assert np.array_equal(gu.bits(heads[j]), want[j])
    # the bulk kernels' own waits all completed
    assert rr.bulk_wait_timeouts(reset=True) == 0
