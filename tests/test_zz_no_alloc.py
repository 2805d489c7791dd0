"""The allocation-free probe (st_probe_noalloc) against the probe that the
search reports (st_search_ex), on two calls in a row sharing the library's fixed
scratch array, plus its host-side size limit.

Collected last on purpose: it must also pass after every other test has run
in the same process."""
import numpy as np
import pytest
import torch

import filtered_int8_ann_b200 as st
import oracle
from workloads import small, to_numpy

pytestmark = pytest.mark.gpu

CASES = [
    # several centroid slices per query (B = 4, nlist = 4096)
    dict(n=20000, d=64, nlist=4096, sig_bits=64, B=4, nprobe=64, k=100, seed=71),
    # one slice per query (B >= 296)
    dict(n=20000, d=128, nlist=512, sig_bits=128, B=400, nprobe=32, k=50, seed=72),
    # nprobe = 4096 over 33000 lists: the centroid keys spill to the fixed
    # array in global memory
    dict(n=20000, d=64, nlist=33000, sig_bits=64, B=4, nprobe=4096, k=20, seed=73),
]


def _oracle_probe(a, rows, P):
    return np.stack([oracle.probe(a["queries"][r], a["centroids"], P) for r in rows])


def _probe_of_search(idx, g, nprobe, k):
    B = g.queries.shape[0]
    probe = torch.empty((B, nprobe), dtype=torch.int32, device="cuda")
    idx.search(g.queries, g.masks, nprobe, k, probe=probe)
    assert idx.check() == st.ST_OK
    return probe.cpu().numpy()


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c['B']}_nlist{c['nlist']}_P{c['nprobe']}")
def test_noalloc_probe_matches_search_two_calls(case):
    data = small(**case)
    g = data.to(torch.device("cuda"))
    P, k, B = case["nprobe"], case["k"], case["B"]
    idx = st.Index(g.items, g.sigs, g.offsets, g.centroids)
    try:
        expected = _probe_of_search(idx, g, P, k)
        out1 = torch.full((B, P), -7, dtype=torch.int32, device="cuda")
        out2 = torch.full((B, P), -7, dtype=torch.int32, device="cuda")
        idx.probe_noalloc(g.queries, P, out1)
        idx.probe_noalloc(g.queries, P, out2)  # same stream, same scratch
        assert idx.check() == st.ST_OK
        assert np.array_equal(out1.cpu().numpy(), expected)
        assert np.array_equal(out2.cpu().numpy(), expected)
        # a smaller request right after reuses the array from whatever the
        # previous call left there
        half = max(1, B // 2)
        out3 = torch.full((half, P), -7, dtype=torch.int32, device="cuda")
        idx.probe_noalloc(g.queries[:half].contiguous(), P, out3)
        assert idx.check() == st.ST_OK
        assert np.array_equal(out3.cpu().numpy(), expected[:half])
    finally:
        idx.close()


def test_noalloc_probe_matches_oracle():
    case = CASES[0]
    data = small(**case)
    g = data.to(torch.device("cuda"))
    P = case["nprobe"]
    a = to_numpy(data)
    exp = _oracle_probe(a, range(case["B"]), P)
    idx = st.Index(g.items, g.sigs, g.offsets, g.centroids)
    try:
        out = torch.empty((case["B"], P), dtype=torch.int32, device="cuda")
        idx.probe_noalloc(g.queries, P, out)
        assert idx.check() == st.ST_OK
        assert np.array_equal(out.cpu().numpy(), exp)
    finally:
        idx.close()


def test_noalloc_probe_rejects_requests_beyond_its_scratch():
    # B = 300 over 20000 lists needs 300 * 20000 * 8 bytes of centroid keys
    data = small(n=5000, d=64, nlist=20000, B=300, nprobe=8, k=10, seed=74)
    g = data.to(torch.device("cuda"))
    idx = st.Index(g.items, g.sigs, g.offsets, g.centroids)
    try:
        out = torch.full((300, 8), -7, dtype=torch.int32, device="cuda")
        with pytest.raises(st.StError) as ei:
            idx.probe_noalloc(g.queries, 8, out)
        assert ei.value.status == st.ST_ERR_SCRATCH_LIMIT
        torch.cuda.synchronize()
        assert bool((out == -7).all())  # nothing was enqueued
        # a smaller batch of the same index fits and is exact
        out_small = torch.empty((40, 8), dtype=torch.int32, device="cuda")
        idx.probe_noalloc(g.queries[:40].contiguous(), 8, out_small)
        assert idx.check() == st.ST_OK
        a = to_numpy(data)
        assert np.array_equal(out_small.cpu().numpy(), _oracle_probe(a, range(40), 8))
    finally:
        idx.close()


def test_noalloc_probe_leaves_free_device_memory_unchanged():
    # Every index, input and output exists before the first reading; after one
    # warm-up call per case (the first call on a device looks up the array's
    # address and sets the kernel's shared-memory limit), repeated calls of
    # every case -- the spill of centroid keys into the array included -- must
    # not change the device's free memory as the driver reports it. The
    # library does not allocate through torch, so torch's own counters would
    # not show an allocation; cudaMemGetInfo does.
    built = []
    try:
        for case in CASES:
            g = small(**case).to(torch.device("cuda"))
            idx = st.Index(g.items, g.sigs, g.offsets, g.centroids)
            out = torch.empty((case["B"], case["nprobe"]), dtype=torch.int32, device="cuda")
            built.append((idx, g, case["nprobe"], out))
        for idx, g, P, out in built:
            idx.probe_noalloc(g.queries, P, out)
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        for _ in range(5):
            for idx, g, P, out in built:
                idx.probe_noalloc(g.queries, P, out)
        torch.cuda.synchronize()
        free1 = torch.cuda.mem_get_info()[0]
        for idx, _, _, _ in built:
            assert idx.check() == st.ST_OK
        assert free1 == free0, f"free device memory changed by {free0 - free1} bytes"
    finally:
        for idx, _, _, _ in built:
            idx.close()
