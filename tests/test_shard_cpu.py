"""Document sharding without a GPU: the row split, the shard offsets, and the
exactness of merging per-shard top-k lists, checked with the CPU oracle on two
gloo ranks (each rank searches its own shard; the ranks gather their top-k
lists and merge them; the result must equal the oracle on the whole index)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from filtered_int8_ann_b200.shard import shard_bounds, shard_offsets  # noqa: E402


def test_bounds_tile_the_rows():
    for n, G in [(12, 3), (10, 4), (7, 7), (100003, 8)]:
        b = [shard_bounds(n, G, g) for g in range(G)]
        assert b[0][0] == 0 and b[-1][1] == n
        assert all(b[i][1] == b[i + 1][0] for i in range(G - 1))
    with pytest.raises(ValueError):
        shard_bounds(10, 2, 2)


def test_offsets_clip_lists_to_the_range():
    off = torch.tensor([0, 3, 3, 10, 12])
    assert shard_offsets(off, 0, 4).tolist() == [0, 3, 3, 4, 4]
    assert shard_offsets(off, 4, 8).tolist() == [0, 0, 0, 4, 4]
    assert shard_offsets(off, 8, 12).tolist() == [0, 0, 0, 2, 4]


def _merge_np(ids, sc, k):
    """Reference merge on the host: k best of the union by (score desc, id asc)."""
    B = ids.shape[1]
    out_i = np.full((B, k), -1, np.int64)
    out_s = np.full((B, k), np.iinfo(np.int32).min, np.int32)
    for b in range(B):
        i = ids[:, b].reshape(-1)
        s = sc[:, b].reshape(-1)
        keep = i >= 0
        i, s = i[keep], s[keep]
        o = np.lexsort((i, -s.astype(np.int64)))[:k]
        out_i[b, :o.size], out_s[b, :o.size] = i[o], s[o]
    return out_i, out_s


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import oracle
    from workloads import small, to_numpy
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        data = small(n=6000, d=32, nlist=24, B=6, nprobe=6, k=300, seed=41, centroid_zipf=0.8)
        a = to_numpy(data)
        n = a["items"].shape[0]
        r0, r1 = shard_bounds(n, world, rank)
        off = shard_offsets(torch.from_numpy(a["offsets"]), r0, r1).numpy()
        ids, sc, _, _ = oracle.search(a["items"][r0:r1], a["sigs"][r0:r1], off, a["centroids"], a["queries"],
                                      a["masks"], 6, 300, nthreads=2)
        ids = np.where(ids >= 0, ids + r0, -1)
        gi = [torch.empty(ids.shape, dtype=torch.int64) for _ in range(world)]
        gs = [torch.empty(sc.shape, dtype=torch.int32) for _ in range(world)]
        dist.all_gather(gi, torch.from_numpy(ids))
        dist.all_gather(gs, torch.from_numpy(sc))
        mi, ms = _merge_np(torch.stack(gi).numpy(), torch.stack(gs).numpy(), 300)
        exp = oracle.search(a["items"], a["sigs"], a["offsets"], a["centroids"], a["queries"], a["masks"], 6, 300,
                            nthreads=2)
        out[rank] = bool(np.array_equal(mi, exp[0]) and np.array_equal(ms, exp[1]))
    finally:
        dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_two_shards_gathered_and_merged_equal_the_whole_index():
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(2, _free_port(), out), nprocs=2, start_method="spawn", join=True)
    assert dict(out) == {0: True, 1: True}
