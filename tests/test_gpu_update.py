"""Streaming in-place updates: replace rows and/or signatures of existing
items (and so their bit-planes), search, and compare bit for bit with the
oracle run on the updated arrays."""
import numpy as np
import pytest
import torch

import filtered_int8_ann_b200 as st
import oracle
from workloads import small, to_numpy

pytestmark = pytest.mark.gpu


def _oracle(a, P, k):
    return oracle.search(a["items"], a["sigs"], a["offsets"], a["centroids"], a["queries"], a["masks"], P, k,
                         nthreads=oracle.max_threads())


@pytest.mark.parametrize("sig_bits,what", [(128, "both"), (128, "sigs"), (64, "rows"), (64, "both")])
def test_update_then_search_matches_oracle(sig_bits, what):
    data = small(n=20000, d=64, nlist=32, sig_bits=sig_bits, hash_bits=3, B=16, nprobe=8, k=300, seed=51,
                 centroid_zipf=0.8)
    donor = small(n=20000, d=64, nlist=32, sig_bits=sig_bits, hash_bits=3, B=16, nprobe=8, k=300, seed=52)
    g = data.to(torch.device("cuda"))
    a = to_numpy(data)
    rng = np.random.default_rng(7)
    m = 3000
    ids = rng.choice(a["items"].shape[0], m, replace=False).astype(np.int64)
    src = rng.choice(donor.items.shape[0], m, replace=False)
    new_items = donor.items.numpy()[src] if what in ("both", "rows") else None
    new_sigs = to_numpy(donor)["sigs"][src] if what in ("both", "sigs") else None
    idx = st.Index(g.items, g.sigs, g.offsets, g.centroids)
    try:
        before, _ = idx.search(g.queries, g.masks, 8, 300)
        idx.update(torch.from_numpy(ids).cuda(),
                   None if new_items is None else torch.from_numpy(new_items).cuda(),
                   None if new_sigs is None else torch.from_numpy(new_sigs.view(np.int64)).cuda())
        ids_got, sc_got = idx.search(g.queries, g.masks, 8, 300)
        assert idx.check() == st.ST_OK
    finally:
        idx.close()
    if new_items is not None:
        a["items"][ids] = new_items
    if new_sigs is not None:
        a["sigs"][ids] = new_sigs
    exp = _oracle(a, 8, 300)
    assert np.array_equal(ids_got.cpu().numpy(), exp[0])
    assert np.array_equal(sc_got.cpu().numpy(), exp[1])
    assert not np.array_equal(before.cpu().numpy(), exp[0])  # the update did change results


def test_update_rejects_bad_arguments_and_records_bad_ids():
    data = small(n=3000, d=32, nlist=8, B=4, nprobe=4, k=50, seed=53)
    g = data.to(torch.device("cuda"))
    idx = st.Index(g.items, g.sigs, g.offsets, g.centroids)
    try:
        ids = torch.tensor([5, 3000, 7], dtype=torch.int64, device="cuda")  # 3000 is out of range
        with pytest.raises(st.StError):
            idx.update(ids)  # neither rows nor signatures
        rows = g.items[:3].clone()
        idx.update(ids, rows)
        assert idx.check() == st.ST_ERR_DEVICE
        assert idx.check() == st.ST_OK
    finally:
        idx.close()
