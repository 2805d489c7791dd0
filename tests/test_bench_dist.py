"""The benchmark's multi-rank plumbing on CPU: two gloo ranks check the
max-over-ranks time, the whole-job sums, and that the ranks search disjoint
query batches drawn from one generated set (replicas: no collective on the
data path)."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    from workloads import small
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        t_max = bench.allreduce_max(float(rank + 1) * 1.5, world, device="cpu")
        q_sum = bench.allreduce_sum(float(10 * (rank + 1)), world, device="cpu")
        B, pool = 3, 2
        data = small(n=500, d=16, nlist=4, B=B * pool * world, seed=5)
        r0, r1 = bench.rank_query_rows(rank, B, pool)
        mine = data.queries[r0:r1]
        gathered = [torch.empty_like(mine) for _ in range(world)]
        dist.all_gather(gathered, mine)
        out[rank] = (t_max, q_sum, (r0, r1),
                     bool(torch.equal(torch.cat(gathered), data.queries[: B * pool * world])))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reductions_and_query_split():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    assert sorted(out.keys()) == [0, 1]
    for r in range(world):
        t_max, q_sum, rows, covers = out[r]
        assert t_max == 3.0          # the slowest rank's time
        assert q_sum == 30.0         # 10 + 20
        assert covers                # the ranks' batches tile the generated set, in rank order
    assert out[0][2] == (0, 6) and out[1][2] == (6, 12)
