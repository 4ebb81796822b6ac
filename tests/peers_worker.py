"""One rank of the two-process, one-GPU run of the one-rank-per-GPU path.

Started by tests/test_gpu_peers.py with RANK, WORLD_SIZE, MASTER_ADDR and
MASTER_PORT set.  Every process drives cuda:0; each keeps only its own rank's
inputs, maps the other's buffers with CUDA IPC (``peers.PeerBuffers``, gloo
for the exchange and the barriers) and computes its own rank's share with
the ``*_rank`` calls.  No kernel waits on another process: the host barriers
order every read after the writes it depends on.  Prints one JSON line and
exits 0 when every check holds."""
import datetime
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

import ragged_reduce_b200 as rr  # noqa: E402
import workloads as wl  # noqa: E402
from ragged_reduce_b200 import peers  # noqa: E402


def same(a, b):
    return a.shape == b.shape and torch.equal(a.contiguous().view(torch.int16),
                                              b.contiguous().view(torch.int16))


def main():
    rank = int(os.environ["RANK"])
    world = int(os.environ["WORLD_SIZE"])
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    T, P, H, D, C = 3001, 3, 56, 128, 2048  # ragged over 2 and 3 ranks
    part = rr.partition(T, H, world)
    ts, te = int(part.token_starts[rank]), int(part.token_starts[rank + 1])
    hs, he = int(part.head_starts[rank]), int(part.head_starts[rank + 1])
    window = max(part.tokens(0) * H * D * 2, T * part.heads(0) * D * 2)
    checks = {}
    tables = []

    # the same seeded bytes in every process; each keeps its own rows
    x = wl.random_bits((T, P, H, D), 7, dev)
    mine = x[ts:te].clone()
    seq_tab = peers.PeerBuffers(mine)
    tables.append(seq_tab)
    head = torch.empty((T, P, he - hs, D), dtype=torch.bfloat16, device=dev)
    torch.cuda.synchronize()
    dist.barrier()
    rr.seq_to_head_rank(seq_tab.pointers, head, rank, n_heads=H, window_bytes=window)
    torch.cuda.synchronize()
    checks["seq_to_head"] = same(head, x[:, :, hs:he, :])

    head_tab = peers.PeerBuffers(head)
    tables.append(head_tab)
    dist.barrier()
    back = torch.empty_like(mine)
    rr.head_to_seq_rank(head_tab.pointers, back, rank, n_tokens=T)
    torch.cuda.synchronize()
    checks["head_to_seq"] = same(back, mine)

    parts = wl.normal_bf16((world, T, C), 11, 0.5, dev)
    bias = wl.normal_bf16((C,), 12, 0.1, dev)
    my_partial = parts[rank].clone()
    part_tab = peers.PeerBuffers(my_partial)
    tables.append(part_tab)
    rs_part = rr.partition(T, world, world)
    rs0, rs1 = int(rs_part.token_starts[rank]), int(rs_part.token_starts[rank + 1])
    out = torch.empty((rs1 - rs0, C), dtype=torch.bfloat16, device=dev)
    torch.cuda.synchronize()
    dist.barrier()
    rr.ragged_reduce_scatter_rank(part_tab.pointers, bias, out, rank, n_tokens=T)
    torch.cuda.synchronize()
    acc = parts[0].float()
    for k in range(1, world):
        acc += parts[k].float()
    acc += bias.float()
    expect = acc.to(torch.bfloat16)
    checks["reduce_scatter"] = same(out, expect[rs0:rs1])

    # gated, in place on this rank's residual rows
    S = 5
    gate = wl.normal_bf16((S, C), 13, 1.0, dev)
    bounds = wl.segment_bounds(T, S, 14)
    x_res = wl.normal_bf16((T, C), 15, 1.0, dev)
    x_mine = x_res[rs0:rs1].clone()
    rr.ragged_reduce_scatter_gated_rank(part_tab.pointers, bias, gate, bounds, x_mine, rank,
                                        n_tokens=T)
    torch.cuda.synchronize()
    seg = torch.from_numpy(np.searchsorted(np.asarray(bounds), np.arange(T), side="right") - 1)
    g_rows = gate.index_select(0, seg.to(dev))
    gated = (x_res.float() + g_rows.float() * expect.float()).to(torch.bfloat16)
    checks["gated"] = same(x_mine, gated[rs0:rs1])

    out_tab = peers.PeerBuffers(out)
    tables.append(out_tab)
    dist.barrier()
    gathered = torch.empty((T, C), dtype=torch.bfloat16, device=dev)
    rr.ragged_all_gather_rank(out_tab.pointers, gathered, rank)
    torch.cuda.synchronize()
    checks["all_gather"] = same(gathered, expect)

    dist.barrier()  # every rank's reads of the others' buffers are done
    for tab in tables:
        tab.close()
    dist.barrier()
    dist.destroy_process_group()
    ok = all(checks.values())
    print(json.dumps({"rank": rank, "ok": ok, **checks}))
    return 0 if ok else 1


if __name__ == "__main__":
    sys.exit(main())
