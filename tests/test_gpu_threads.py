"""Calls from several host threads at once.  The library keeps per-device
caches behind locks and each thread's last CUDA error on its own; nothing
else is shared, so concurrent calls on separate streams must each give the
oracle's result.  The GPU case runs tests/threads_worker.py in a fresh
process so that the threads also race to fill the cold caches; the host
plan (h3_partition) is checked concurrently on the CPU."""
import os
import subprocess
import sys
import threading

import numpy as np
import pytest

import ragged_reduce_b200 as rr

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.gpu
def test_threads_on_their_own_streams():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "threads_worker.py")],
                         cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert out.returncode == 0, out.stdout[-3000:] + out.stderr[-3000:]
    assert "threads ok" in out.stdout


def test_partition_from_many_threads(oracle_lib):
    """16 threads, 100 plans each, against the oracle's partition and clip."""
    errors = []
    start = threading.Barrier(16)

    def run(seed):
        rng = np.random.default_rng(seed)
        try:
            start.wait(timeout=60)
            for _ in range(100):
                T = int(rng.integers(64, 100_000))
                W = int(rng.integers(1, 65))
                H = int(rng.integers(W, 200))
                S = int(rng.integers(1, 33))
                cuts = np.sort(rng.choice(np.arange(1, T), size=S - 1, replace=False))
                bounds = np.concatenate([[0], cuts, [T]]).astype(np.int64)
                p = rr.partition(T, H, W, bounds)
                if not (np.array_equal(p.token_starts, oracle_lib.partition_range(T, W)) and
                        np.array_equal(p.head_starts.astype(np.int64),
                                       oracle_lib.partition_range(H, W))):
                    errors.append((seed, T, H, W, "ranges"))
                    return
                for r in range(W):
                    lb, ids = oracle_lib.clip_segments(bounds, int(p.token_starts[r]),
                                                       int(p.token_starts[r + 1]))
                    if not (np.array_equal(p.local_bounds[r], lb) and
                            np.array_equal(p.seg_ids[r], ids)):
                        errors.append((seed, T, W, r, "pieces"))
                        return
        except Exception as e:  # noqa: BLE001 - reported below
            errors.append((seed, repr(e)))

    threads = [threading.Thread(target=run, args=(100 + i,)) for i in range(16)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not errors, errors[:5]
