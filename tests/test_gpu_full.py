"""GPU parity at full workload sizes, in the configuration the benchmark times:
the CUDA results are compared bit for bit with the CPU oracle on every query
of the 80M-item Zipf IVF, the flat 10M scan and the 10M batch sweep at every
batch size (B = 1, 8, 64, 256, 1024)."""
import numpy as np
import pytest
import torch

import filtered_int8_ann_b200 as st
import oracle
from workloads import SWEEP_BATCHES, WORKLOADS, generate, to_numpy

pytestmark = pytest.mark.gpu


def _oracle_rows(a, queries, masks, P, k, rows):
    nt = oracle.max_threads()
    ids = np.empty((len(rows), k), np.int64)
    sc = np.empty((len(rows), k), np.int32)
    el = np.empty(len(rows), np.int64)
    qs = np.ascontiguousarray(queries[rows])
    ms = np.ascontiguousarray(masks[rows])
    r = oracle.search(a["items"], a["sigs"], a["offsets"], a["centroids"], qs, ms, P, k, nthreads=nt)
    return r[0], r[1], r[2], r[3]


def _search(idx, q, m, P, k):
    B = q.shape[0]
    elig = torch.empty(B, dtype=torch.int64, device="cuda")
    probe = torch.empty((B, P), dtype=torch.int32, device="cuda")
    ids, sc = idx.search(q, m, P, k, eligible=elig, probe=probe)
    assert idx.check() == st.ST_OK
    return ids.cpu().numpy(), sc.cpu().numpy(), probe.cpu().numpy(), elig.cpu().numpy()


def _check(got, exp, rows, what):
    for g, e, n in zip(got, exp, ("ids", "scores", "probe", "eligible")):
        g = g[rows]
        assert np.array_equal(g, e), f"{what}: {n} differ"


def _run(name, batches=None):
    wl = WORKLOADS[name]
    data = generate(wl, device="cuda")
    idx = st.Index(data.items, data.sigs, data.offsets, data.centroids)
    a = to_numpy(data)
    try:
        for B in batches or (wl.B,):
            q = data.queries[:B].contiguous()
            m = data.masks[:B].contiguous()
            got = _search(idx, q, m, wl.nprobe, wl.k)
            rows = np.arange(B)
            exp = _oracle_rows(a, a["queries"][:B], a["masks"][:B], wl.nprobe, wl.k, rows)
            _check(got, exp, rows, f"{name} B={B}")
            if B == (batches or (wl.B,))[-1]:
                again = _search(idx, q, m, wl.nprobe, wl.k)
                for x, y in zip(got, again):
                    assert np.array_equal(x, y), "repeat differs"
    finally:
        idx.close()


def test_full_ivf_80m_all_queries():
    _run("ivf_80m")


def test_full_flat_10m():
    _run("flat_10m")


def test_full_sweep_10m_batches():
    _run("sweep_10m", batches=SWEEP_BATCHES)
