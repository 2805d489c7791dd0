"""OR of several masks per query (Index.search_any: one search per alternative
and st_merge_topk_union) against two expected values that must agree: the
oracle run once per alternative, its lists united by the plain definition
(every item of the union's top-k is in the top-k of each alternative it
passes), and an independent numpy brute force that tests every alternative on
every item of the probed lists."""
import numpy as np
import pytest
import torch

import bruteforce as bf
import filtered_int8_ann_b200 as st
import oracle
from workloads import small, to_numpy

pytestmark = pytest.mark.gpu


def _bf_search_any(a, mask_sets, P, k):
    B = a["queries"].shape[0]
    ids = np.full((B, k), -1, np.int64)
    sc = np.full((B, k), bf.INT32_MIN, np.int32)
    for b in range(B):
        lists = bf.probe(a["queries"][b], a["centroids"], P)
        rows = np.concatenate([np.arange(a["offsets"][c], a["offsets"][c + 1]) for c in lists])
        ok = np.zeros(rows.size, bool)
        for ms in mask_sets:
            ok |= bf.bloom_pass(a["sigs"][rows], ms[b])
        rows = rows[ok]
        if rows.size == 0:
            continue
        s = bf.scores(a["queries"][b][None, :], a["items"][rows])[0]
        o = bf.order_desc(s, rows)[:k]
        ids[b, :o.size], sc[b, :o.size] = rows[o], s[o]
    return ids, sc


def _oracle_search_any(a, mask_sets, P, k):
    per = [oracle.search(a["items"], a["sigs"], a["offsets"], a["centroids"], a["queries"], np.ascontiguousarray(ms),
                         P, k, nthreads=oracle.max_threads()) for ms in mask_sets]
    B = a["queries"].shape[0]
    ids = np.full((B, k), -1, np.int64)
    sc = np.full((B, k), np.iinfo(np.int32).min, np.int32)
    for b in range(B):
        pairs = {}
        for r in per:
            for i, s in zip(r[0][b], r[1][b]):
                if i >= 0:
                    pairs[int(i)] = int(s)
        best = sorted(pairs.items(), key=lambda t: (-t[1], t[0]))[:k]
        for j, (i, s) in enumerate(best):
            ids[b, j], sc[b, j] = i, s
    return ids, sc


@pytest.mark.parametrize("sig_bits", [64, 128])
def test_or_of_masks_matches_brute_force(sig_bits):
    data = small(n=15000, d=32, nlist=24, sig_bits=sig_bits, hash_bits=3, B=8, nprobe=6, k=200, seed=81,
                 mask_country=True, mask_flags=3)
    other = small(n=15000, d=32, nlist=24, sig_bits=sig_bits, hash_bits=3, B=8, nprobe=6, k=200, seed=82,
                  mask_mode="item", mask_country=True, mask_flags=1)
    a = to_numpy(data)
    m2 = to_numpy(other)["masks"]
    m3 = a["masks"].copy()
    m3[:, 0] &= np.uint64(0xFF)  # fewer required bits: a looser alternative
    sets = [a["masks"], m2, m3]
    g = data.to(torch.device("cuda"))
    mask_sets = torch.from_numpy(np.stack(sets).view(np.int64)).cuda()
    idx = st.Index(g.items, g.sigs, g.offsets, g.centroids)
    try:
        ids, sc = idx.search_any(g.queries, mask_sets, 6, 200)
        assert idx.check() == st.ST_OK
        assert st.st_merge_check() == st.ST_OK
        # one alternative twice: the union is the plain search
        same = torch.stack([mask_sets[0], mask_sets[0]])
        i2, s2 = idx.search_any(g.queries, same, 6, 200)
        i1, s1 = idx.search(g.queries, g.masks, 6, 200)
    finally:
        idx.close()
    exp = _oracle_search_any(a, sets, 6, 200)
    brute = _bf_search_any(a, sets, 6, 200)
    assert np.array_equal(exp[0], brute[0]) and np.array_equal(exp[1], brute[1])
    assert np.array_equal(ids.cpu().numpy(), exp[0]) and np.array_equal(sc.cpu().numpy(), exp[1])
    assert np.array_equal(i2.cpu().numpy(), i1.cpu().numpy()) and np.array_equal(s2.cpu().numpy(), s1.cpu().numpy())
