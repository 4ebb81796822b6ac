"""Worker for tests/test_gpu_threads.py: several host threads in a fresh
process (every per-device cache of the library still cold: SM count,
resident CTAs, shared-memory opt-ins) start together, and each drives its own
mix of calls on its own CUDA stream and buffers for ten rounds.  Every round
first overwrites the outputs with a canary on that stream, then calls, then
compares the outputs with the oracle's.  Prints "threads ok" and exits 0
when every check holds."""
import os
import sys
import threading
import traceback

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import oracle  # noqa: E402
import ragged_reduce_b200 as rr  # noqa: E402
import workloads as wl  # noqa: E402

DEV = "cuda"
ROUNDS = 10
CANARY = 0x7FC1


def _bits(t):
    return wl.bf16_bits(t)


def _on_device(arrays):
    return [torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(DEV) for a in arrays]


class Job:
    """Outputs to check (device tensors) and their expected 16-bit patterns."""

    name = "job"

    def outputs(self):
        raise NotImplementedError

    def calls(self, stream):
        raise NotImplementedError

    def round(self, stream):
        with torch.cuda.stream(stream):
            for t in self.outputs():
                t.view(torch.int16).fill_(CANARY)
        self.calls(stream)

    def mismatches(self):
        return [i for i, (t, e) in enumerate(zip(self.outputs(), self.expected))
                if not torch.equal(t.contiguous().view(torch.int16).view(-1), e.view(-1))]


class Relayout(Job):
    def __init__(self, o, seed, T, P, H, D, W, window=0, variant=0, token_chunks=False):
        self.name = (f"relayout T={T} P={P} W={W} window={window} variant={variant}"
                     f"{' token ranges' if token_chunks else ''}")
        self.window, self.variant, self.token_chunks = window, variant, token_chunks
        full = wl.random_bits((T, P, H, D), seed, DEV)
        part = rr.partition(T, H, W)
        self.send = rr.split_rows(full, part.token_starts)
        self.heads = rr.alloc_head_side(T, P, H, D, W, DEV)
        _, self.back = rr.alloc_seq_side(T, P, H, D, W, DEV)
        want = o.seq_to_head([_bits(s) for s in self.send], T, P, H, D, W)
        self.expected = _on_device(want) + _on_device([_bits(s) for s in self.send])

    def outputs(self):
        return self.heads + self.back

    def calls(self, stream):
        rr.seq_to_head(self.send, self.heads, window_bytes=self.window, variant=self.variant,
                       stream=stream, token_chunks=self.token_chunks)
        rr.head_to_seq(self.heads, self.back, window_bytes=self.window, variant=self.variant,
                       stream=stream, token_chunks=self.token_chunks)


class Staged(Relayout):
    def __init__(self, o, seed, T, P, H, D, W, window_rows):
        super().__init__(o, seed, T, P, H, D, W)
        self.name = f"staged T={T} P={P} W={W} window={window_rows} rows"
        self.win = torch.empty(window_rows * H * D * 2, dtype=torch.uint8, device=DEV)

    def calls(self, stream):
        rr.seq_to_head_staged(self.send, self.heads, self.win, stream=stream)
        rr.head_to_seq_staged(self.heads, self.back, self.win, stream=stream)


class ReduceGather(Job):
    def __init__(self, o, seed, T, C, W, ctas_per_sm=0, gather_variant=0):
        self.name = f"reduce+gather T={T} C={C} W={W}"
        self.ctas_per_sm, self.gather_variant = ctas_per_sm, gather_variant
        self.partials = wl.normal_bf16((W, T, C), seed, 0.5, DEV)
        self.bias = wl.normal_bf16((C,), seed + 1, 0.1, DEV)
        _, self.red = rr.alloc_reduce_outputs(T, C, W, DEV)
        self.gath = [torch.empty((T, C), dtype=torch.bfloat16, device=DEV) for _ in range(W)]
        red = o.ragged_reduce_scatter([_bits(p) for p in self.partials.unbind(0)], _bits(self.bias), W)
        self.expected = _on_device(red) + _on_device(o.ragged_all_gather(red, W))

    def outputs(self):
        return self.red + self.gath

    def calls(self, stream):
        rr.ragged_reduce_scatter(self.partials, self.bias, self.red, stream=stream,
                                 ctas_per_sm=self.ctas_per_sm)
        rr.ragged_all_gather(self.red, self.gath, stream=stream, variant=self.gather_variant)


class Gated(Job):
    def __init__(self, o, seed, T, C, W, S):
        self.name = f"gated T={T} C={C} W={W} S={S}"
        self.partials = wl.normal_bf16((W, T, C), seed, 0.5, DEV)
        self.bias = wl.normal_bf16((C,), seed + 1, 0.1, DEV)
        self.gate = wl.normal_bf16((S, C), seed + 2, 1.0, DEV)
        self.bounds = wl.segment_bounds(T, S, seed + 3)
        part = rr.partition(T, W, W)
        self.x = rr.split_rows(wl.normal_bf16((T, C), seed + 4, 1.0, DEV), part.token_starts)
        _, self.out = rr.alloc_reduce_outputs(T, C, W, DEV)
        want = o.reduce_scatter_gated([_bits(p) for p in self.partials.unbind(0)], _bits(self.bias),
                                      _bits(self.gate), self.bounds, [_bits(v) for v in self.x], W)
        self.expected = _on_device(want)

    def outputs(self):
        return self.out

    def calls(self, stream):
        rr.ragged_reduce_scatter_gated(self.partials, self.bias, self.gate, self.bounds, self.x,
                                       self.out, stream=stream)


def main():
    o = oracle.load()
    jobs = [
        Relayout(o, 401, 1000, 3, 56, 128, 6),
        Relayout(o, 402, 777, 4, 56, 128, 8, window=700_000),  # 3 token chunks per plane
        Relayout(o, 403, 513, 1, 56, 128, 4, variant=rr.H3_VARIANT_BULK),
        # bulk kernels over token ranges of all three planes (5 ranges)
        Relayout(o, 404, 1000, 3, 56, 128, 6, window=1_700_000, variant=rr.H3_VARIANT_BULK,
                 token_chunks=True),
        Staged(o, 405, 600, 3, 56, 128, 5, window_rows=41),
        ReduceGather(o, 406, 1000, 7168, 6),
        ReduceGather(o, 407, 333, 7168, 3, ctas_per_sm=2, gather_variant=rr.H3_VARIANT_BULK),
        Gated(o, 408, 777, 2048, 8, 5),
    ]
    torch.cuda.synchronize()
    start = threading.Barrier(len(jobs))
    errors = []

    def run(job):
        try:
            stream = torch.cuda.Stream()
            start.wait(timeout=120)
            for rnd in range(ROUNDS):
                job.round(stream)
                stream.synchronize()
                bad = job.mismatches()
                if bad:
                    errors.append(f"{job.name}, round {rnd}: outputs {bad} differ from the oracle")
                    return
        except Exception:
            errors.append(f"{job.name}: {traceback.format_exc()}")

    threads = [threading.Thread(target=run, args=(j,), daemon=True) for j in jobs]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
        if t.is_alive():
            errors.append("a thread did not finish within 300 s")
    if errors:
        print("\n".join(errors))
        sys.exit(1)
    print("threads ok")


if __name__ == "__main__":
    main()
