"""Host-side row map of the library (where inserted items go, and the chunk
table the search walks), compiled from the library's own header into a small
host-only shim and checked against an independent Python model of the layout
rule: creation rows first; each list's new items fill its last append chunk in
call order, then a fresh chunk numbered after every earlier one; an item's id
is its row."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def shim(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("index_map") / "libindex_map_shim.so")
    subprocess.run(["g++", "-std=c++17", "-O1", "-Wall", "-Werror", "-shared", "-fPIC",
                    os.path.join(HERE, "index_map_shim.cpp"), "-o", out], check=True)
    L = ctypes.CDLL(out)
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    L.im_create.argtypes, L.im_create.restype = [P, i32, i32], P
    L.im_place.argtypes, L.im_place.restype = [P, P, i64, i64, i64, P], i32
    L.im_app_used.argtypes, L.im_app_used.restype = [P], i32
    L.im_build.argtypes, L.im_build.restype = [P], i32
    L.im_tables.argtypes, L.im_tables.restype = [P, P, P, P, P], None
    L.im_destroy.argtypes, L.im_destroy.restype = [P], None
    return L


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


class Model:
    """The layout rule restated: per list, the current append chunk and its fill."""

    def __init__(self, off, chunk):
        self.n, self.chunk, self.nlist = int(off[-1]), chunk, len(off) - 1
        self.last = {}        # list -> its last append chunk
        self.fill = []        # append chunk -> rows filled
        self.members = {c: [] for c in range(self.nlist)}  # inserted ids per list, in order

    def place(self, lists):
        ids = []
        for L in lists:
            a = self.last.get(int(L))
            if a is None or self.fill[a] == self.chunk:
                a = len(self.fill)
                self.fill.append(0)
                self.last[int(L)] = a
            ids.append(self.n + self.chunk * a + self.fill[a])
            self.fill[a] += 1
            self.members[int(L)].append(ids[-1])
        return np.array(ids, dtype=np.int64)


def _offsets(rng, nlist, sizes_max):
    sizes = rng.integers(0, sizes_max, nlist)
    sizes[rng.choice(nlist, max(1, nlist // 5), replace=False)] = 0  # some empty lists
    sizes[0] = max(sizes[0], 1)
    return np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)


def _place(shim, h, lists, id_offset=0, id_limit=2**31):
    lists = np.ascontiguousarray(lists, dtype=np.int32)
    ids = np.empty(len(lists), dtype=np.int64)
    ok = shim.im_place(h, _p(lists), len(lists), id_offset, id_limit, _p(ids))
    return bool(ok), ids


def _tables(shim, h, nlist):
    nd = shim.im_build(h)
    desc = np.empty((nd, 4), dtype=np.int32)
    start = np.empty(nlist + 1, dtype=np.int32)
    top_rows = np.empty(nlist + 1, dtype=np.int64)
    top_chunks = np.empty(nlist + 1, dtype=np.int64)
    shim.im_tables(h, _p(desc), _p(start), _p(top_rows), _p(top_chunks))
    return desc, start, top_rows, top_chunks


@pytest.mark.parametrize("chunk,nlist,sizes_max,seed", [(512, 37, 3000, 1), (4, 9, 11, 2), (16, 1, 50, 3)])
def test_ids_and_chunk_table_follow_the_layout_rule(shim, chunk, nlist, sizes_max, seed):
    rng = np.random.default_rng(seed)
    off = _offsets(rng, nlist, sizes_max)
    h = shim.im_create(_p(off), nlist, chunk)
    try:
        model = Model(off, chunk)
        for m in (1, 7, 3 * chunk + 1, 200, 2 * chunk, 0, 5):
            lists = rng.integers(0, nlist, m).astype(np.int32)
            if m > 4:
                lists[: m // 2] = rng.integers(0, nlist)  # one list takes a run
            ok, ids = _place(shim, h, lists)
            assert ok
            assert np.array_equal(ids, model.place(lists))
        assert shim.im_app_used(h) == len(model.fill)
        desc, start, top_rows, top_chunks = _tables(shim, h, nlist)
        n, nb = int(off[-1]), 0
        base_blocks = []
        for c in range(nlist):
            nc = int(off[c + 1] - off[c])
            base_blocks.append(nb)
            nb += -(-nc // chunk)
        sizes, counts = [], []
        for c in range(nlist):
            ent = desc[start[c]:start[c + 1]]
            assert np.all(ent[:, 3] == c) and np.all(ent[:, 2] >= 1) and np.all(ent[:, 2] <= chunk)
            rows = np.concatenate([np.arange(r, r + k) for r, _, k, _ in ent]) if len(ent) else np.zeros(0, np.int64)
            expect = np.concatenate([np.arange(off[c], off[c + 1]), model.members[c]]).astype(np.int64)
            assert np.array_equal(rows, expect), c
            ncre = -(-int(off[c + 1] - off[c]) // chunk)
            assert list(ent[:ncre, 1]) == list(range(base_blocks[c], base_blocks[c] + ncre))
            for r, blk, k, _ in ent[ncre:]:
                a = (r - n) // chunk
                assert (r - n) % chunk == 0 and blk == nb + a and k == model.fill[a]
            sizes.append(len(expect))
            counts.append(len(ent))
        assert start[0] == 0 and start[-1] == len(desc)
        assert np.array_equal(top_rows, np.concatenate([[0], np.cumsum(sorted(sizes, reverse=True))]))
        assert np.array_equal(top_chunks, np.concatenate([[0], np.cumsum(sorted(counts, reverse=True))]))
    finally:
        shim.im_destroy(h)


def test_placement_refused_at_the_id_limit_changes_nothing(shim):
    off = np.array([0, 10, 10, 25], dtype=np.int64)
    h = shim.im_create(_p(off), 3, 8)
    try:
        model = Model(off, 8)
        ok, ids = _place(shim, h, [0, 0, 2])
        assert ok and np.array_equal(ids, model.place([0, 0, 2]))
        # rows 25..40 are handed out (two chunks); a third chunk would end at
        # row 49, which with an id offset of 100 reaches a limit of 149
        ok, _ = _place(shim, h, [1] * 3, id_offset=100, id_limit=149)
        assert not ok
        assert shim.im_app_used(h) == 2
        # the same request under a higher limit: as if the refused one never happened
        ok, ids = _place(shim, h, [1] * 3, id_offset=100, id_limit=150)
        assert ok and np.array_equal(ids, model.place([1] * 3))
        # filling an existing chunk needs no new room
        ok, ids = _place(shim, h, [0] * 6, id_offset=100, id_limit=150)
        assert ok and np.array_equal(ids, model.place([0] * 6))
    finally:
        shim.im_destroy(h)
