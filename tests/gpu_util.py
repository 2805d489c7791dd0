"""Shared helpers of the GPU parity tests: run the CUDA library and the CPU
oracle on the same seeded inputs."""
import numpy as np
import torch

import filtered_int8_ann_b200 as st
import oracle
from workloads import to_numpy


def run_gpu(data, nprobe, k, index=None, cap=None, stream=None):
    dev = torch.device("cuda")
    g = data.to(dev) if data.items.device.type != "cuda" else data
    own = index is None
    if own:
        index = st.Index(g.items, g.sigs, g.offsets, g.centroids)
    try:
        if cap is not None:
            index.set_option(st.ST_OPT_CANDIDATE_CAPACITY, cap)
        B = g.queries.shape[0]
        elig = torch.empty(B, dtype=torch.int64, device=dev)
        probe = torch.empty((B, nprobe), dtype=torch.int32, device=dev)
        ids, sc = index.search(g.queries, g.masks, nprobe, k, eligible=elig, probe=probe, stream=stream)
        assert index.check(stream) == st.ST_OK
        return ids.cpu().numpy(), sc.cpu().numpy(), probe.cpu().numpy(), elig.cpu().numpy()
    finally:
        if own:
            index.close()


def run_oracle(data, nprobe, k, b0=0, b1=None, nthreads=None):
    a = to_numpy(data)
    nthreads = nthreads or oracle.max_threads()
    return oracle.search(a["items"], a["sigs"], a["offsets"], a["centroids"], a["queries"], a["masks"],
                         nprobe, k, b0=b0, b1=b1, nthreads=nthreads)


def assert_parity(got, exp, what=""):
    names = ("ids", "scores", "probe", "eligible")
    for g, e, n in zip(got, exp, names):
        if not np.array_equal(g, e):
            bad = np.argwhere(g != e) if g.shape == e.shape else None
            raise AssertionError(f"{what} {n} differ (shape {g.shape} vs {e.shape}); first bad {bad[:5] if bad is not None else ''}")
