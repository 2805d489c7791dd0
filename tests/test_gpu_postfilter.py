"""Deleted items (st_index_delete) and per-query exclude masks
(st_search_extras.exclude_masks) leave the final top-k before selection. The
expected results come from the CPU oracle run on signatures where the removed
items can no longer pass: every mask here is non-zero, so a zero signature
never passes it."""
import numpy as np
import pytest
import torch

import filtered_int8_ann_b200 as st
import oracle
from workloads import bloom_words, small, to_numpy

pytestmark = pytest.mark.gpu


def _oracle(a, P, k, sigs=None, rows=None):
    qs, ms = a["queries"], a["masks"]
    if rows is not None:
        qs, ms = np.ascontiguousarray(qs[rows]), np.ascontiguousarray(ms[rows])
    return oracle.search(a["items"], a["sigs"] if sigs is None else sigs, a["offsets"], a["centroids"], qs, ms,
                         P, k, nthreads=oracle.max_threads())


def _search(idx, g, P, k, exclude=None):
    ids, sc = idx.search(g.queries, g.masks, P, k, exclude=exclude)
    assert idx.check() == st.ST_OK
    return ids.cpu().numpy(), sc.cpu().numpy()


def _exclude_oracle(a, P, k, x):
    """Per query: items holding every bit of its exclude mask get a zero signature."""
    out_i, out_s = [], []
    for b in range(a["queries"].shape[0]):
        sg = a["sigs"].copy()
        if x[b].any():
            hit = np.all((sg & x[b]) == x[b], axis=1)
            sg[hit] = 0
        r = _oracle(a, P, k, sigs=sg, rows=[b])
        out_i.append(r[0][0])
        out_s.append(r[1][0])
    return np.stack(out_i), np.stack(out_s)


CASE = dict(n=20000, d=64, nlist=32, sig_bits=128, hash_bits=3, B=12, nprobe=8, k=300, seed=71, centroid_zipf=0.8)


def test_deleted_items_never_return():
    data = small(**CASE)
    a = to_numpy(data)
    assert np.all(a["masks"].any(axis=1))
    g = data.to(torch.device("cuda"))
    idx = st.Index(g.items, g.sigs, g.offsets, g.centroids)
    try:
        first, _ = _search(idx, g, 8, 300)
        rng = np.random.default_rng(3)
        gone = np.unique(np.concatenate([first[0, :100], rng.choice(20000, 2000, replace=False)]))
        gone = gone[gone >= 0].astype(np.int64)
        idx.delete(torch.from_numpy(gone).cuda())
        idx.delete(torch.from_numpy(gone[:10]).cuda())  # twice is harmless
        ids, sc = _search(idx, g, 8, 300)
        idx.delete(torch.tensor([20000], dtype=torch.int64, device="cuda"))  # outside the index
        assert idx.check() == st.ST_ERR_DEVICE
        assert idx.check() == st.ST_OK
    finally:
        idx.close()
    sg = a["sigs"].copy()
    sg[gone] = 0
    exp = _oracle(a, 8, 300, sigs=sg)
    assert np.array_equal(ids, exp[0]) and np.array_equal(sc, exp[1])
    assert not np.isin(ids, gone).any()


@pytest.mark.parametrize("k,cap", [(300, None), (300, 1400), (6000, None)])
def test_exclude_masks(k, cap):
    # "not flag 3" for even queries, nothing excluded for odd ones
    data = small(**CASE)
    a = to_numpy(data)
    flag3 = np.array(bloom_words(0xB10057 + CASE["seed"], 2 + 3, 1, 128, 3), dtype=np.uint64)
    x = np.zeros_like(a["masks"])
    x[0::2] = flag3
    g = data.to(torch.device("cuda"))
    idx = st.Index(g.items, g.sigs, g.offsets, g.centroids)
    try:
        if cap is not None:
            idx.set_option(st.ST_OPT_CANDIDATE_CAPACITY, cap)  # forces the exact overflow rescan
        ids, sc = _search(idx, g, 8, k, exclude=torch.from_numpy(x.view(np.int64)).cuda())
    finally:
        idx.close()
    exp = _exclude_oracle(a, 8, k, x)
    assert np.array_equal(ids, exp[0]) and np.array_equal(sc, exp[1])


def test_deletion_with_one_crowded_bin():
    # every score equal: the cut bin holds every candidate, more than the kept tie list
    data = small(n=20000, d=16, nlist=2, sig_bits=64, B=2, nprobe=2, k=3000, seed=72, mask_flags=1,
                 mask_lang=False)
    data.items[:] = 2
    a = to_numpy(data)
    assert np.all(a["masks"].any(axis=1))
    g = data.to(torch.device("cuda"))
    idx = st.Index(g.items, g.sigs, g.offsets, g.centroids)
    try:
        gone = np.arange(0, 20000, 3, dtype=np.int64)
        idx.delete(torch.from_numpy(gone).cuda())
        ids, sc = _search(idx, g, 2, 3000)
    finally:
        idx.close()
    sg = a["sigs"].copy()
    sg[gone] = 0
    exp = _oracle(a, 2, 3000, sigs=sg)
    assert np.array_equal(ids, exp[0]) and np.array_equal(sc, exp[1])
