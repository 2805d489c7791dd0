"""Insertion of new items into existing IVF lists (st_index_insert), alone and
mixed with in-place updates and deletions, compared bit for bit with the CPU
oracle run on the equivalent index: each list's creation rows followed by the
items inserted into it, with the ids the library returned as item ids."""
import numpy as np
import pytest
import torch

import filtered_int8_ann_b200 as st
import oracle
from workloads import small, to_numpy

pytestmark = pytest.mark.gpu

CHUNK = st.ST_INSERT_CHUNK


class Mirror:
    """Host copy of an index under insertions, updates and deletions: item id ->
    (list, row, signature); rebuilt into CSR arrays for the oracle."""

    def __init__(self, a):
        self.a = a
        off = a["offsets"]
        self.list_of = {}
        self.row = {}
        self.sig = {}
        for c in range(len(off) - 1):
            for i in range(off[c], off[c + 1]):
                self.list_of[i] = c
                self.row[i] = a["items"][i]
                self.sig[i] = a["sigs"][i]

    def insert(self, lists, items, sigs, ids):
        for L, x, s, i in zip(lists, items, sigs, ids):
            assert int(i) not in self.list_of
            self.list_of[int(i)] = int(L)
            self.row[int(i)] = x
            self.sig[int(i)] = s

    def update(self, ids, items=None, sigs=None):
        for j, i in enumerate(ids):
            if items is not None:
                self.row[int(i)] = items[j]
            if sigs is not None:
                self.sig[int(i)] = sigs[j]

    def delete(self, ids):
        for i in ids:
            self.list_of.pop(int(i), None)

    def csr(self):
        nlist = self.a["centroids"].shape[0]
        by_list = [[] for _ in range(nlist)]
        for i, L in self.list_of.items():
            by_list[L].append(i)
        # any order inside a list: the oracle orders by the ids
        ids = np.array([i for L in range(nlist) for i in by_list[L]], dtype=np.int64)
        off = np.zeros(nlist + 1, dtype=np.int64)
        off[1:] = np.cumsum([len(v) for v in by_list])
        items = np.stack([self.row[i] for i in ids]).astype(np.int8)
        sigs = np.stack([self.sig[i] for i in ids]).astype(np.uint64)
        return items, sigs, off, ids

    def search(self, P, k, rows=None):
        items, sigs, off, ids = self.csr()
        qs, ms = self.a["queries"], self.a["masks"]
        if rows is not None:
            qs, ms = np.ascontiguousarray(qs[rows]), np.ascontiguousarray(ms[rows])
        return oracle.search(items, sigs, off, self.a["centroids"], qs, ms, P, k, nthreads=oracle.max_threads(),
                             row_ids=ids)


def _insert_batch(idx, mirror, donor, lists, rng):
    m = len(lists)
    src = rng.choice(donor["items"].shape[0], m, replace=False)
    items = np.ascontiguousarray(donor["items"][src])
    sigs = np.ascontiguousarray(donor["sigs"][src])
    ids = idx.insert(lists, torch.from_numpy(items).cuda(), torch.from_numpy(sigs.view(np.int64)).cuda())
    assert idx.check() == st.ST_OK
    mirror.insert(lists, items, sigs, ids)
    return ids


def _insert_query_twins(idx, mirror, a):
    """One item per query equal to the query vector, with every signature bit
    set, in the query's best list: it scores |q|^2 and passes any mask, so it
    must appear in that query's results."""
    qs = a["queries"]
    lists = np.array([oracle.probe(q, a["centroids"], 1)[0] for q in qs], np.int32)
    sigs = np.full((qs.shape[0], a["sigs"].shape[1]), np.uint64(2**64 - 1), np.uint64)
    ids = idx.insert(lists, torch.from_numpy(np.ascontiguousarray(qs)).cuda(),
                     torch.from_numpy(sigs.view(np.int64)).cuda())
    assert idx.check() == st.ST_OK
    mirror.insert(lists, qs, sigs, ids)
    return ids


def _search(idx, g, P, k):
    ids, sc = idx.search(g.queries, g.masks, P, k)
    assert idx.check() == st.ST_OK
    return ids.cpu().numpy(), sc.cpu().numpy()


def _same(got, exp):
    assert np.array_equal(got[0], exp[0])
    assert np.array_equal(got[1], exp[1])


def _skewed_lists(rng, nlist, m, hot, hot_count):
    lists = rng.integers(0, nlist, m).astype(np.int32)
    lists[rng.choice(m, hot_count, replace=False)] = hot
    return lists


@pytest.mark.parametrize("sig_bits", [64, 128])
def test_insert_then_search_matches_oracle(sig_bits):
    kw = dict(n=20000, d=64, nlist=32, sig_bits=sig_bits, hash_bits=3, B=16, nprobe=8, k=300)
    data = small(seed=81, centroid_zipf=0.8, **kw)
    donor = to_numpy(small(seed=82, **kw))
    a = to_numpy(data)
    g = data.to(torch.device("cuda"))
    rng = np.random.default_rng(83)
    mirror = Mirror(a)
    idx = st.Index(g.items, g.sigs, g.offsets, g.centroids)
    try:
        _same(_search(idx, g, 8, 300), mirror.search(8, 300))
        # one list takes 1500 rows (three append chunks), the rest spread out
        lists = _skewed_lists(rng, 32, 3000, hot=int(np.argmax(np.diff(a["offsets"]))), hot_count=1500)
        ids = _insert_batch(idx, mirror, donor, lists, rng)
        twins = _insert_query_twins(idx, mirror, a)
        assert len(np.unique(ids)) == len(ids) and ids.min() >= 20000
        # a list's items fill its chunks in argument order
        for L in np.unique(lists):
            own = ids[lists == L]
            assert np.all(np.diff(own) > 0)
            assert np.all(own[1:][np.diff(own) != 1] % CHUNK == 20000 % CHUNK)
        got = _search(idx, g, 8, 300)
        _same(got, mirror.search(8, 300))
        # the new items do take part: each query finds its twin
        assert all(twins[b] in got[0][b] for b in range(len(twins)))
    finally:
        idx.close()


def test_insert_batches_grow_update_delete_large_k():
    kw = dict(n=12000, d=32, nlist=24, sig_bits=128, hash_bits=2, B=8, nprobe=6, k=200)
    data = small(seed=84, **kw)
    donor = to_numpy(small(seed=85, **kw))
    a = to_numpy(data)
    g = data.to(torch.device("cuda"))
    rng = np.random.default_rng(86)
    mirror = Mirror(a)
    idx = st.Index(g.items, g.sigs, g.offsets, g.centroids)
    try:
        all_ids = []
        # batches of growing size: the append room is reallocated several times
        for m in (1, 40, 700, 2500, 5000):
            lists = _skewed_lists(rng, 24, m, hot=3, hot_count=m // 2)
            all_ids.append(_insert_batch(idx, mirror, donor, lists, rng))
            if m == 40:
                all_ids.append(_insert_query_twins(idx, mirror, a))
            _same(_search(idx, g, 6, 200), mirror.search(6, 200))
        new = np.concatenate(all_ids)
        # update some inserted rows (rows and signatures) and some creation rows
        up = np.concatenate([rng.choice(new, 300, replace=False), rng.choice(12000, 100, replace=False)])
        src = rng.choice(donor["items"].shape[0], len(up), replace=False)
        ui, us = np.ascontiguousarray(donor["items"][src]), np.ascontiguousarray(donor["sigs"][src])
        idx.update(torch.from_numpy(up).cuda(), torch.from_numpy(ui).cuda(), torch.from_numpy(us.view(np.int64)).cuda())
        mirror.update(up, ui, us)
        # delete some of the best results, inserted or not
        first = _search(idx, g, 6, 200)[0]
        gone = np.unique(np.concatenate([first[:, :20].ravel(), rng.choice(new, 500, replace=False)]))
        gone = gone[gone >= 0].astype(np.int64)
        idx.delete(torch.from_numpy(gone).cuda())
        mirror.delete(gone)
        _same(_search(idx, g, 6, 200), mirror.search(6, 200))
        # k above the shared-memory final top-k: room sized with the inserted rows
        _same(_search(idx, g, 6, 9000), mirror.search(6, 9000))
        # one more batch after deletions, into a list no query may probe first
        _insert_batch(idx, mirror, donor, np.full(600, 7, np.int32), rng)
        _same(_search(idx, g, 6, 200), mirror.search(6, 200))
    finally:
        idx.close()


def test_insert_overflow_path_walks_append_chunks():
    kw = dict(n=10000, d=64, nlist=16, sig_bits=64, hash_bits=2, B=6, nprobe=4, k=100)
    data = small(seed=87, mask_flags=0, **kw)
    donor = to_numpy(small(seed=88, mask_flags=0, **kw))
    a = to_numpy(data)
    g = data.to(torch.device("cuda"))
    rng = np.random.default_rng(89)
    mirror = Mirror(a)
    idx = st.Index(g.items, g.sigs, g.offsets, g.centroids)
    try:
        _insert_batch(idx, mirror, donor, _skewed_lists(rng, 16, 4000, hot=5, hot_count=2000), rng)
        twins = _insert_query_twins(idx, mirror, a)
        # a candidate buffer of k + 1024 keys: busy queries take the exact rescan
        idx.set_option(st.ST_OPT_CANDIDATE_CAPACITY, 1)
        got = _search(idx, g, 4, 100)
        _same(got, mirror.search(4, 100))
        assert all(twins[b] in got[0][b] for b in range(len(twins)))
        idx.set_option(st.ST_OPT_CANDIDATE_CAPACITY, 0)
        _same(_search(idx, g, 4, 100), mirror.search(4, 100))
    finally:
        idx.close()


def test_insert_rejections_leave_the_index_unchanged():
    kw = dict(n=6000, d=32, nlist=8, sig_bits=64, B=4, nprobe=4, k=50)
    data = small(seed=90, **kw)
    donor = to_numpy(small(seed=91, **kw))
    a = to_numpy(data)
    g = data.to(torch.device("cuda"))
    rng = np.random.default_rng(92)
    mirror = Mirror(a)
    idx = st.Index(g.items, g.sigs, g.offsets, g.centroids)
    try:
        items = torch.from_numpy(np.ascontiguousarray(donor["items"][:3])).cuda()
        sigs = torch.from_numpy(np.ascontiguousarray(donor["sigs"][:3]).view(np.int64)).cuda()
        for bad in ([0, 8, 1], [-1, 0, 0]):
            with pytest.raises(st.StError) as ei:
                idx.insert(np.array(bad, np.int32), items, sigs)
            assert ei.value.status == st.ST_ERR_INVALID_ARG
        with pytest.raises(st.StError) as ei:  # host rows are not device memory
            idx.insert(np.array([0, 1, 2], np.int32), items.cpu(), sigs)
        assert ei.value.status == st.ST_ERR_INVALID_ARG
        _same(_search(idx, g, 4, 50), mirror.search(4, 50))
        # ids would pass 2^31 with the id offset: refused, nothing changes
        idx.set_option(st.ST_OPT_ID_OFFSET, 2**31 - 6000 - 100)
        with pytest.raises(st.StError) as ei:
            idx.insert(np.array([0, 1, 2], np.int32), items, sigs)
        assert ei.value.status == st.ST_ERR_UNSUPPORTED
        idx.set_option(st.ST_OPT_ID_OFFSET, 0)
        _same(_search(idx, g, 4, 50), mirror.search(4, 50))
        # room reserved up front, then used without a reallocation
        idx.set_option(st.ST_OPT_INSERT_RESERVE, 3 * CHUNK)
        _insert_batch(idx, mirror, donor, np.full(3 * CHUNK, 2, np.int32), rng)
        _same(_search(idx, g, 4, 50), mirror.search(4, 50))
        # an id inside an append chunk that no insertion handed out yet is refused
        hole = torch.tensor([6000 + 3 * CHUNK + 5], dtype=torch.int64, device="cuda")
        ids = _insert_batch(idx, mirror, donor, np.array([4], np.int32), rng)
        assert ids[0] == 6000 + 3 * CHUNK
        idx.update(hole, items[:1])
        assert idx.check() == st.ST_ERR_DEVICE
        assert idx.check() == st.ST_OK
        _same(_search(idx, g, 4, 50), mirror.search(4, 50))
    finally:
        idx.close()


def test_insert_with_id_offset_and_search_host():
    kw = dict(n=8000, d=64, nlist=12, sig_bits=128, hash_bits=3, B=5, nprobe=5, k=64)
    data = small(seed=93, **kw)
    donor = to_numpy(small(seed=94, **kw))
    a = to_numpy(data)
    g = data.to(torch.device("cuda"))
    rng = np.random.default_rng(95)
    mirror = Mirror(a)
    idx = st.Index(g.items, g.sigs, g.offsets, g.centroids)
    try:
        idx.set_option(st.ST_OPT_ID_OFFSET, 1000000)
        _insert_batch(idx, mirror, donor, rng.integers(0, 12, 1500).astype(np.int32), rng)
        _insert_query_twins(idx, mirror, a)
        exp = mirror.search(5, 64)
        assert (exp[0] >= 8000).any()
        ids, sc = idx.search_host(torch.from_numpy(a["queries"]), torch.from_numpy(a["masks"].view(np.int64)), 5, 64)
        shifted = np.where(exp[0] >= 0, exp[0] + 1000000, -1)
        assert np.array_equal(ids.numpy(), shifted)
        assert np.array_equal(sc.numpy(), exp[1])
    finally:
        idx.close()
