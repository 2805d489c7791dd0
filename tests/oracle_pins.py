"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Every pin takes a loaded oracle library (the real one, or a mutant build with a
planted mistake) and raises AssertionError when the oracle disagrees with:
hand-worked cases from the definition (tests/golden/*.json), closed forms,
special cases, or the independent numpy restatement in bruteforce.py.
"""
import json
import os

import numpy as np

import bruteforce
import oracle
from workloads import small

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
INT32_MIN = -2**31


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _one_list(n, d):
    return np.array([0, n], dtype=np.int64), np.zeros((1, d), dtype=np.int8)


def _axis_items(values, d=16):
    """Items whose score against the query e_0 equals the given values."""
    x = np.zeros((len(values), d), dtype=np.int8)
    x[:, 0] = values
    q = np.zeros((1, d), dtype=np.int8)
    q[0, 0] = 1
    return x, q


# --- step 1/3: inner products ---------------------------------------------------
def pin_dot_library(lib):
    rng = np.random.default_rng(11)
    for d in (16, 48, 64, 128, 512):
        for _ in range(20):
            a = rng.integers(-128, 128, d, dtype=np.int8)
            b = rng.integers(-128, 128, d, dtype=np.int8)
            assert oracle.dot(a, b, lib) == int(a.astype(np.int64) @ b.astype(np.int64)), d


def pin_dot_extremes(lib):
    for d in (16, 64, 128, 512):
        hi = np.full(d, 127, np.int8)
        lo = np.full(d, -128, np.int8)
        assert oracle.dot(hi, hi, lib) == d * 127 * 127
        assert oracle.dot(lo, lo, lib) == d * 128 * 128
        assert oracle.dot(hi, lo, lib) == -d * 127 * 128
        alt = np.array([127, -128] * (d // 2), np.int8)
        assert oracle.dot(alt, hi, lib) == (d // 2) * (127 * 127 - 128 * 127)


# --- step 2: probe ---------------------------------------------------------------
def pin_probe_golden(lib):
    g = golden("probe_ties.json")
    cent, q = _axis_items(g["centroid_scores"])
    got = oracle.probe(q[0], cent, g["nprobe"], lib)
    assert list(got) == g["expect_lists"], got


def pin_probe_all_equal(lib):
    rng = np.random.default_rng(3)
    row = rng.integers(-128, 128, 32, dtype=np.int8)
    cent = np.tile(row, (40, 1))
    q = rng.integers(-128, 128, 32, dtype=np.int8)
    for P in (1, 7, 40):
        assert list(oracle.probe(q, cent, P, lib)) == list(range(P))


def pin_probe_full_and_library(lib):
    rng = np.random.default_rng(5)
    for nlist, d in ((1, 16), (13, 16), (64, 32), (300, 64)):
        # few distinct values so that ties are common
        cent = rng.integers(-2, 3, (nlist, d), dtype=np.int8)
        for _ in range(5):
            q = rng.integers(-3, 4, d, dtype=np.int8)
            full = oracle.probe(q, cent, nlist, lib)
            assert sorted(full) == list(range(nlist))
            assert np.array_equal(full, bruteforce.probe(q, cent, nlist))
            P = max(1, nlist // 3)
            assert np.array_equal(oracle.probe(q, cent, P, lib), full[:P])


# --- step 3: Bloom eligibility -----------------------------------------------------
def pin_bloom_golden(lib):
    for c in golden("bloom_cases.json")["cases"]:
        sig = np.array([int(w, 16) for w in c["sig"]], dtype=np.uint64)
        mask = np.array([int(w, 16) for w in c["mask"]], dtype=np.uint64)
        assert oracle.bloom_pass(sig, mask, lib) == c["pass"], c["why"]


def pin_bloom_special(lib):
    rng = np.random.default_rng(9)
    for W in (1, 2):
        sigs = rng.integers(0, 2**63, (200, W), dtype=np.uint64) | rng.integers(0, 2, (200, W), dtype=np.uint64) << np.uint64(63)
        sigs[7] = np.uint64(2**64 - 1)
        zero = np.zeros(W, np.uint64)
        ones = np.full(W, 2**64 - 1, np.uint64)
        for i in range(200):
            assert oracle.bloom_pass(sigs[i], zero, lib)
            assert oracle.bloom_pass(sigs[i], sigs[i], lib)
            assert oracle.bloom_pass(sigs[i], ones, lib) == bool(np.all(sigs[i] == ones))
            m = sigs[(i * 31 + 1) % 200]
            assert oracle.bloom_pass(sigs[i], m, lib) == bool(bruteforce.bloom_pass(sigs[i:i + 1], m)[0])


# --- step 4: top-k order and padding -------------------------------------------------
def _search_axis(lib, values, k, eligible=None):
    x, q = _axis_items(values)
    n = len(values)
    off, cen = _one_list(n, x.shape[1])
    sigs = np.ones((n, 1), np.uint64) if eligible is None else \
        np.array([[1 if e else 0] for e in eligible], np.uint64)
    masks = np.ones((1, 1), np.uint64)
    ids, sc, _, _ = oracle.search(x, sigs, off, cen, q, masks, 1, k, lib=lib)
    return ids[0], sc[0]


def pin_topk_golden(lib):
    g = golden("topk_ties.json")
    ids, sc = _search_axis(lib, g["scores"], g["k"])
    assert list(ids) == g["expect_ids"] and list(sc) == g["expect_scores"], (ids, sc)


def pin_padding_golden(lib):
    g = golden("padding.json")
    ids, sc = _search_axis(lib, g["scores"], g["k"], g["eligible"])
    assert list(ids) == g["expect_ids"] and list(sc) == g["expect_scores"], (ids, sc)


def pin_topk_identical(lib):
    rng = np.random.default_rng(2)
    row = rng.integers(-128, 128, 32, dtype=np.int8)
    x = np.tile(row, (300, 1))
    q = rng.integers(-128, 128, (1, 32), dtype=np.int8)
    off, cen = _one_list(300, 32)
    sigs = np.zeros((300, 1), np.uint64)
    masks = np.zeros((1, 1), np.uint64)
    ids, sc, _, el = oracle.search(x, sigs, off, cen, q, masks, 1, 100, lib=lib)
    s = int(row.astype(np.int64) @ q[0].astype(np.int64))
    assert list(ids[0]) == list(range(100)) and np.all(sc[0] == s) and el[0] == 300


# --- whole search ---------------------------------------------------------------------
def _arrays(data):
    from workloads import to_numpy
    return to_numpy(data)


def pin_ivf_full_probe_equals_flat(lib):
    for seed, W in ((21, 1), (22, 2)):
        data = small(n=1500, d=32, nlist=12, sig_bits=64 * W, B=6, nprobe=12, k=200, seed=seed)
        a = _arrays(data)
        f = _arrays(data.flat())
        ivf = oracle.search(a["items"], a["sigs"], a["offsets"], a["centroids"], a["queries"],
                            a["masks"], 12, 200, lib=lib)
        flat = oracle.search(f["items"], f["sigs"], f["offsets"], f["centroids"], f["queries"],
                             f["masks"], 1, 200, lib=lib)
        assert np.array_equal(ivf[0], flat[0]) and np.array_equal(ivf[1], flat[1])
        assert np.array_equal(ivf[3], flat[3])


def pin_bruteforce_tiny(lib):
    cases = [
        dict(n=400, d=16, nlist=4, sig_bits=64, B=5, nprobe=2, k=30, seed=31),
        dict(n=2000, d=64, nlist=16, sig_bits=128, hash_bits=3, B=6, nprobe=5, k=64, seed=32,
             mask_country=True),
        dict(n=1200, d=128, nlist=8, sig_bits=128, B=4, nprobe=8, k=1500, seed=33),
        dict(n=900, d=48, nlist=30, sig_bits=64, B=7, nprobe=1, k=7, seed=34, mask_flags=0,
             mask_lang=False),
        dict(n=1000, d=32, nlist=10, sig_bits=64, B=5, nprobe=3, k=40, seed=35,
             mask_mode="item", mask_country=True),
        dict(n=1500, d=16, nlist=1, sig_bits=128, B=3, nprobe=1, k=100, seed=36,
             uniform_items=True),
        dict(n=1800, d=32, nlist=24, sig_bits=128, B=8, nprobe=6, k=90, seed=37,
             centroid_zipf=0.8),
    ]
    for c in cases:
        data = small(**c)
        a = _arrays(data)
        P, k = c["nprobe"], c["k"]
        got = oracle.search(a["items"], a["sigs"], a["offsets"], a["centroids"], a["queries"],
                            a["masks"], P, k, lib=lib)
        exp = bruteforce.search(a["items"], a["sigs"], a["offsets"], a["centroids"],
                                a["queries"], a["masks"], P, k)
        for g, e, what in zip(got, exp, ("ids", "scores", "probe", "eligible")):
            assert np.array_equal(g, e), (c, what)


def pin_threads_do_not_change_result(lib):
    data = small(n=2000, d=32, nlist=16, B=12, nprobe=5, k=60, seed=41)
    a = _arrays(data)
    r1 = oracle.search(a["items"], a["sigs"], a["offsets"], a["centroids"], a["queries"],
                       a["masks"], 5, 60, nthreads=1, lib=lib)
    r4 = oracle.search(a["items"], a["sigs"], a["offsets"], a["centroids"], a["queries"],
                       a["masks"], 5, 60, nthreads=4, lib=lib)
    for x, y in zip(r1, r4):
        assert np.array_equal(x, y)


def pin_sub_batch(lib):
    data = small(n=1000, d=32, nlist=8, B=9, nprobe=3, k=20, seed=43)
    a = _arrays(data)
    full = oracle.search(a["items"], a["sigs"], a["offsets"], a["centroids"], a["queries"],
                         a["masks"], 3, 20, lib=lib)
    part = oracle.search(a["items"], a["sigs"], a["offsets"], a["centroids"], a["queries"],
                         a["masks"], 3, 20, b0=4, b1=7, lib=lib)
    for x, y in zip(full, part):
        assert np.array_equal(x[4:7], y)


# --- explicit item ids per row (an index whose lists took insertions) -------------------
def _permute_within_lists(a, rng):
    """Rows of each list in a random order, with the original row index as the id."""
    off = a["offsets"]
    perm = np.concatenate([off[c] + rng.permutation(off[c + 1] - off[c]) for c in range(len(off) - 1)])
    return a["items"][perm], a["sigs"][perm], perm.astype(np.int64)


def pin_row_ids_permutation(lib):
    """Reordering the rows inside each list, each keeping its item id, leaves
    the result unchanged; repeated rows make every score tie, so only the ids
    order them."""
    rng = np.random.default_rng(61)
    for c in (dict(n=1500, d=32, nlist=10, sig_bits=128, B=6, nprobe=4, k=120, seed=62),
              dict(n=800, d=16, nlist=3, sig_bits=64, B=4, nprobe=2, k=900, seed=63)):
        a = _arrays(small(**c))
        P, k = c["nprobe"], c["k"]
        exp = oracle.search(a["items"], a["sigs"], a["offsets"], a["centroids"], a["queries"], a["masks"], P, k,
                            lib=lib)
        items, sigs, ids = _permute_within_lists(a, rng)
        got = oracle.search(items, sigs, a["offsets"], a["centroids"], a["queries"], a["masks"], P, k, lib=lib,
                            row_ids=ids)
        for g, e in zip(got, exp):
            assert np.array_equal(g, e), c
    # all scores equal: the order is the ids' order
    n, d = 300, 16
    x = np.tile(rng.integers(-128, 128, d, dtype=np.int8), (n, 1))
    q = rng.integers(-128, 128, (1, d), dtype=np.int8)
    off, cen = _one_list(n, d)
    ids = rng.permutation(np.arange(1000, 1000 + 3 * n, 3)).astype(np.int64)
    got_ids, got_sc, _, el = oracle.search(x, np.zeros((n, 1), np.uint64), off, cen, q, np.zeros((1, 1), np.uint64),
                                           1, 50, lib=lib, row_ids=ids)
    assert list(got_ids[0]) == list(range(1000, 1150, 3)) and el[0] == n


def pin_row_ids_bruteforce(lib):
    rng = np.random.default_rng(64)
    for c in (dict(n=1200, d=32, nlist=8, sig_bits=128, hash_bits=3, B=5, nprobe=3, k=80, seed=65),
              dict(n=600, d=16, nlist=1, sig_bits=64, B=4, nprobe=1, k=700, seed=66, uniform_items=True)):
        a = _arrays(small(**c))
        n = a["items"].shape[0]
        ids = rng.choice(20 * n, n, replace=False).astype(np.int64)
        P, k = c["nprobe"], c["k"]
        got = oracle.search(a["items"], a["sigs"], a["offsets"], a["centroids"], a["queries"], a["masks"], P, k,
                            lib=lib, row_ids=ids)
        exp = bruteforce.search(a["items"], a["sigs"], a["offsets"], a["centroids"], a["queries"], a["masks"],
                                P, k, row_ids=ids)
        for g, e, what in zip(got, exp, ("ids", "scores", "probe", "eligible")):
            assert np.array_equal(g, e), (c, what)


# --- step 3 with alternative masks (an OR of values) ---------------------------------
def pin_or_golden(lib):
    g = golden("or_masks.json")
    x, q = _axis_items(g["scores"])
    n = len(g["scores"])
    off, cen = _one_list(n, x.shape[1])
    sigs = np.array(g["sigs"], np.uint64).reshape(n, 1)
    for order in (1, -1):  # the result does not depend on the order of the alternatives
        ms = np.array(g["masks"][::order], np.uint64).reshape(1, -1, 1)
        ids, sc, _, el = oracle.search_or(x, sigs, off, cen, q, ms, 1, g["k"], lib=lib)
        assert list(ids[0]) == g["expect_ids"] and list(sc[0]) == g["expect_scores"], (ids, sc)
        assert int(el[0]) == g["expect_eligible"], el


def _or_cases():
    rng = np.random.default_rng(71)
    out = []
    for c in (dict(n=1500, d=32, nlist=8, sig_bits=64, hash_bits=2, B=6, nprobe=3, k=60, seed=72, mask_flags=2),
              dict(n=2000, d=16, nlist=12, sig_bits=128, hash_bits=3, B=5, nprobe=4, k=300, seed=73,
                   mask_country=True, mask_flags=1),
              dict(n=800, d=48, nlist=1, sig_bits=128, B=4, nprobe=1, k=900, seed=74, mask_mode="item")):
        a = _arrays(small(**c))
        B, W = a["masks"].shape
        n = a["sigs"].shape[0]
        # alternatives: the query's own mask, another query's, and the bits of
        # a random item's signature under a random sub-mask
        alt = [a["masks"], np.roll(a["masks"], 1, axis=0),
               a["sigs"][rng.integers(0, n, B)] & rng.integers(0, 2**63, (B, W), dtype=np.uint64)]
        out.append((c, a, np.ascontiguousarray(np.stack(alt, axis=1))))
    return out


def pin_or_bruteforce(lib):
    for c, a, ms in _or_cases():
        P, k = c["nprobe"], c["k"]
        for A in (1, 2, 3):
            got = oracle.search_or(a["items"], a["sigs"], a["offsets"], a["centroids"], a["queries"],
                                   np.ascontiguousarray(ms[:, :A]), P, k, lib=lib)
            exp = bruteforce.search_or(a["items"], a["sigs"], a["offsets"], a["centroids"], a["queries"],
                                       ms[:, :A], P, k)
            for g_, e, what in zip(got, exp, ("ids", "scores", "probe", "eligible")):
                assert np.array_equal(g_, e), (c, A, what)


def pin_or_union_of_single_masks(lib):
    # every item of the union's top-k is in the top-k of each alternative it
    # passes, so merging the single-mask results (distinct ids, score
    # descending, id ascending) gives the OR search's ids and scores
    for c, a, ms in _or_cases():
        P, k = c["nprobe"], c["k"]
        A = ms.shape[1]
        got = oracle.search_or(a["items"], a["sigs"], a["offsets"], a["centroids"], a["queries"], ms, P, k,
                               lib=lib)
        singles = [oracle.search(a["items"], a["sigs"], a["offsets"], a["centroids"], a["queries"],
                                 np.ascontiguousarray(ms[:, j]), P, k, lib=lib) for j in range(A)]
        for b in range(a["queries"].shape[0]):
            pairs = {}
            for r in singles:
                for i, s_ in zip(r[0][b], r[1][b]):
                    if i >= 0:
                        pairs[int(i)] = int(s_)
            best = sorted(pairs.items(), key=lambda t: (-t[1], t[0]))[:k]
            exp_i = [t[0] for t in best] + [-1] * (k - len(best))
            exp_s = [t[1] for t in best] + [INT32_MIN] * (k - len(best))
            assert list(got[0][b]) == exp_i and list(got[1][b]) == exp_s, (c, b)
            assert int(got[3][b]) >= max(int(r[3][b]) for r in singles), (c, b)


PINS = [v for k_, v in sorted(globals().items()) if k_.startswith("pin_")]
