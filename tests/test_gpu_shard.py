"""Document sharding: each shard (a contiguous row range with the index's
centroids and its id offset) is searched as its own index, st_merge_topk merges
the shards' top-k lists, and the result must equal the unsharded search and the
CPU oracle bit for bit."""
import numpy as np
import pytest
import torch

import filtered_int8_ann_b200 as st
from gpu_util import run_oracle
from workloads import WORKLOADS, generate, small

pytestmark = pytest.mark.gpu


def _sharded(g, shards, P, k):
    B = g.queries.shape[0]
    ids = torch.empty((shards, B, k), dtype=torch.int64, device="cuda")
    sc = torch.empty((shards, B, k), dtype=torch.int32, device="cuda")
    for s in range(shards):
        idx = st.Index.shard(g.items, g.sigs, g.offsets, g.centroids, shards, s)
        try:
            idx.search(g.queries, g.masks, P, k, out_ids=ids[s], out_scores=sc[s])
            assert idx.check() == st.ST_OK
        finally:
            idx.close()
    mi, ms = st.st_merge_topk(ids, sc)
    assert st.st_merge_check() == st.ST_OK
    return mi.cpu().numpy(), ms.cpu().numpy()


CASES = [
    (dict(n=20000, d=64, nlist=64, sig_bits=128, hash_bits=3, B=16, nprobe=8, k=256, seed=31,
          centroid_zipf=0.8), 2),
    (dict(n=20000, d=128, nlist=40, sig_bits=64, B=8, nprobe=40, k=1000, seed=32), 3),
    (dict(n=9000, d=64, nlist=10, sig_bits=128, B=5, nprobe=10, k=4096, seed=33, mask_flags=0,
          mask_lang=False), 4),
]


@pytest.mark.parametrize("case,shards", CASES, ids=lambda c: str(c) if isinstance(c, int) else f"n{c['n']}_k{c['k']}")
def test_sharded_search_equals_unsharded_and_oracle(case, shards):
    data = small(**case)
    g = data.to(torch.device("cuda"))
    P, k = case["nprobe"], case["k"]
    got_ids, got_sc = _sharded(g, shards, P, k)
    idx = st.Index(g.items, g.sigs, g.offsets, g.centroids)
    try:
        ids, sc = idx.search(g.queries, g.masks, P, k)
        assert idx.check() == st.ST_OK
    finally:
        idx.close()
    assert np.array_equal(got_ids, ids.cpu().numpy())
    assert np.array_equal(got_sc, sc.cpu().numpy())
    exp = run_oracle(data, P, k)
    assert np.array_equal(got_ids, exp[0]) and np.array_equal(got_sc, exp[1])


def test_sharded_mid_ivf_eight_shards():
    wl = WORKLOADS["mid_ivf"]
    g = generate(wl, device="cuda")
    got_ids, got_sc = _sharded(g, 8, wl.nprobe, wl.k)
    exp = run_oracle(g.to(torch.device("cpu")), wl.nprobe, wl.k)
    assert np.array_equal(got_ids, exp[0]) and np.array_equal(got_sc, exp[1])


def test_merge_rejects_bad_sizes_and_flags_bad_ids():
    ids = torch.full((2, 3, 4), -1, dtype=torch.int64, device="cuda")
    sc = torch.zeros((2, 3, 4), dtype=torch.int32, device="cuda")
    with pytest.raises(st.StError) as e:
        st.st_merge_topk(ids.reshape(1, 6, 4).expand(5000, 6, 4).contiguous(), sc.reshape(1, 6, 4).expand(5000, 6, 4).contiguous())
    assert e.value.status == st.ST_ERR_UNSUPPORTED
    # all padding -> all padding
    oi, osc = st.st_merge_topk(ids, sc)
    assert st.st_merge_check() == st.ST_OK
    assert bool((oi == -1).all()) and bool((osc == torch.iinfo(torch.int32).min).all())
    # an id that is neither valid nor padding is reported
    ids[1, 2, 0] = -5
    st.st_merge_topk(ids, sc)
    assert st.st_merge_check() == st.ST_ERR_DEVICE
    assert st.st_merge_check() == st.ST_OK  # cleared
