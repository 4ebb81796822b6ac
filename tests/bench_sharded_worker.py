"""One rank of bench.py's one-rank-per-GPU step, run as processes that share
one GPU (started by tests/test_gpu_bench_sharded.py with RANK, WORLD_SIZE,
MASTER_ADDR and MASTER_PORT set).

Everything is the bench's own code path except the fence between calls: the
real binding and rank calls, peer tables over real CUDA IPC, CUDA-event
timing, the per-rank check and the end-to-end loop.  The ranks cannot run
NCCL on one GPU, so the fence synchronises the stream and meets the other
ranks in a gloo all-reduce on the host; no kernel waits on another process.
Prints rank 0's bench line (or {"rank": r} on the other ranks) and exits 0."""
import datetime
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

import bench  # noqa: E402
import ragged_reduce_b200 as rr  # noqa: E402
from ragged_reduce_b200 import peers  # noqa: E402

TOKENS, ROWS = 3001, 1000


def main():
    rank = int(os.environ["RANK"])
    world = int(os.environ["WORLD_SIZE"])
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    token = torch.zeros(1)

    def fence(stream=None):
        (stream or torch.cuda.current_stream(dev)).synchronize()
        dist.all_reduce(token)

    def make_step():
        return bench.ShardedStep(dev, rank, world, rr=rr, peer_table=peers.PeerBuffers,
                                 fence=fence, tokens=TOKENS, rows=ROWS)

    args = bench.parse_args(["--gpus", str(world), "--steps", "5", "--warmup", "3",
                             "--e2e-steps", "2"])
    result = bench.measure(args, make_step, rank, world, 0, dev, bench.CudaTimer(), 5)
    torch.cuda.synchronize()
    dist.barrier()
    dist.destroy_process_group()
    print(json.dumps(result if rank == 0 else {"rank": rank}), flush=True)


if __name__ == "__main__":
    main()
