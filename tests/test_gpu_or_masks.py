"""OR of several masks per query. The fused scan (st_search_extras.or_masks,
Index.search_any) is checked against the oracle's OR search on sparse and
dense (tensor-core) units, single-query units, unions wider than the plane
buffers, an all-pass alternative and the exact overflow path; the first test
also checks it against two expected values that must agree: the oracle run
once per alternative, its lists united by the plain definition (every item of
the union's top-k is in the top-k of each alternative it passes), and an
independent numpy brute force that tests every alternative on every item of
the probed lists. The per-alternative merge (search_any_merged) must give the
same result."""
import numpy as np
import pytest
import torch

import bruteforce as bf
import filtered_int8_ann_b200 as st
import oracle
from gpu_util import assert_parity, run_oracle
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


# --- the fused scan: alternative masks tested inside one search ----------------------
def _alternatives(a, rng, A):
    """A masks per query [B, A, W]: the query's own mask, another query's, a
    random item's signature under a random sub-mask, then further random
    sub-masks of items' signatures."""
    B, W = a["masks"].shape
    n = a["sigs"].shape[0]
    alt = [a["masks"], np.roll(a["masks"], 1, axis=0)]
    while len(alt) < A:
        alt.append(a["sigs"][rng.integers(0, n, B)] & rng.integers(0, 2**63, (B, W), dtype=np.uint64))
    return np.ascontiguousarray(np.stack(alt[:A], axis=1))


def _fused(data, ms, P, k, min_q=None, cap=None):
    g = data.to(torch.device("cuda"))
    idx = st.Index(g.items, g.sigs, g.offsets, g.centroids)
    try:
        if min_q is not None:
            idx.set_option(st.ST_OPT_DENSE_MIN_QUERIES, min_q)
        if cap is not None:
            idx.set_option(st.ST_OPT_CANDIDATE_CAPACITY, cap)
        B = g.queries.shape[0]
        qm = torch.from_numpy(np.ascontiguousarray(ms[:, 0]).view(np.int64)).cuda()
        alt = torch.from_numpy(np.ascontiguousarray(ms[:, 1:]).view(np.int64)).cuda() if ms.shape[1] > 1 else None
        elig = torch.empty(B, dtype=torch.int64, device="cuda")
        probe = torch.empty((B, P), dtype=torch.int32, device="cuda")
        ids, sc = idx.search(g.queries, qm, P, k, eligible=elig, probe=probe, or_masks=alt)
        assert idx.check() == st.ST_OK
        return ids.cpu().numpy(), sc.cpu().numpy(), probe.cpu().numpy(), elig.cpu().numpy()
    finally:
        idx.close()


OR_CASES = [
    # sparse units of one and several queries, W = 2 and 1, generic d (no row registers)
    dict(n=20000, d=32, nlist=24, sig_bits=128, hash_bits=3, B=8, nprobe=6, k=200, seed=91, mask_country=True,
         mask_flags=2, A=3),
    dict(n=12000, d=48, nlist=16, sig_bits=64, hash_bits=2, B=5, nprobe=4, k=80, seed=92, mask_flags=2, A=2),
    dict(n=9000, d=64, nlist=12, sig_bits=128, hash_bits=3, B=1, nprobe=5, k=300, seed=93, mask_flags=1, A=4),
    # dense units (tensor cores at the default threshold and when forced), d = 64 and 128
    dict(n=8000, d=64, nlist=4, sig_bits=128, hash_bits=3, B=40, nprobe=3, k=100, seed=94, mask_flags=1,
         mask_lang=False, A=3),
    dict(n=8000, d=128, nlist=5, sig_bits=64, hash_bits=2, B=36, nprobe=4, k=500, seed=95, mask_flags=2, A=2),
    # item-mode masks and many alternatives: unions wider than the plane buffers
    dict(n=10000, d=64, nlist=6, sig_bits=128, hash_bits=3, B=24, nprobe=3, k=150, seed=96, mask_mode="item",
         mask_country=True, mask_flags=3, A=8),
]


@pytest.mark.parametrize("case", OR_CASES, ids=[f"or{i}" for i in range(len(OR_CASES))])
def test_fused_or_matches_oracle(case):
    c = dict(case)
    A = c.pop("A")
    data = small(**c)
    a = to_numpy(data)
    ms = _alternatives(a, np.random.default_rng(c["seed"]), A)
    P, k = c["nprobe"], c["k"]
    exp = oracle.search_or(a["items"], a["sigs"], a["offsets"], a["centroids"], a["queries"], ms, P, k,
                           nthreads=oracle.max_threads())
    for min_q in (None, 1, 0):
        got = _fused(data, ms, P, k, min_q=min_q)
        assert_parity(got, exp, f"{case} dense_min_queries={min_q}")


def test_fused_or_all_pass_alternative_and_single_mask():
    # an all-zero alternative passes every row: the result is the unfiltered
    # search; one alternative equal to the mask: the plain search
    data = small(n=9000, d=64, nlist=8, sig_bits=128, hash_bits=3, B=12, nprobe=3, k=120, seed=97, mask_flags=3)
    a = to_numpy(data)
    zero = np.zeros_like(a["masks"])
    ms = np.ascontiguousarray(np.stack([a["masks"], zero], axis=1))
    exp = oracle.search_or(a["items"], a["sigs"], a["offsets"], a["centroids"], a["queries"], ms, 3, 120,
                           nthreads=oracle.max_threads())
    unf = oracle.search(a["items"], a["sigs"], a["offsets"], a["centroids"], a["queries"], zero, 3, 120,
                        nthreads=oracle.max_threads())
    assert all(np.array_equal(x, y) for x, y in zip(exp, unf))
    for min_q in (1, 0):
        assert_parity(_fused(data, ms, 3, 120, min_q=min_q), exp, f"all-pass alternative min_q={min_q}")
    same = np.ascontiguousarray(np.stack([a["masks"], a["masks"]], axis=1))
    assert_parity(_fused(data, same, 3, 120), run_oracle(data, 3, 120), "repeated mask")


def test_fused_or_overflow_path():
    # a candidate capacity far below the eligible count: every query takes the
    # exact overflow path, which tests the alternatives itself
    data = small(n=20000, d=64, nlist=4, sig_bits=64, hash_bits=2, B=10, nprobe=2, k=64, seed=98, mask_flags=1,
                 mask_lang=False)
    a = to_numpy(data)
    ms = _alternatives(a, np.random.default_rng(98), 3)
    exp = oracle.search_or(a["items"], a["sigs"], a["offsets"], a["centroids"], a["queries"], ms, 2, 64,
                           nthreads=oracle.max_threads())
    assert exp[3].min() > 64 + 1024
    assert_parity(_fused(data, ms, 2, 64, min_q=0, cap=64 + 1024), exp, "overflow path")


def test_fused_or_equals_per_alternative_merge():
    data = small(n=15000, d=32, nlist=24, sig_bits=128, hash_bits=3, B=8, nprobe=6, k=200, seed=99,
                 mask_country=True, mask_flags=3)
    a = to_numpy(data)
    ms = _alternatives(a, np.random.default_rng(99), 3)
    g = data.to(torch.device("cuda"))
    sets = torch.from_numpy(np.ascontiguousarray(ms.transpose(1, 0, 2)).view(np.int64)).cuda()
    idx = st.Index(g.items, g.sigs, g.offsets, g.centroids)
    try:
        i1, s1 = idx.search_any(g.queries, sets, 6, 200)
        i2, s2 = idx.search_any_merged(g.queries, sets, 6, 200)
        assert idx.check() == st.ST_OK
    finally:
        idx.close()
    assert np.array_equal(i1.cpu().numpy(), i2.cpu().numpy()) and np.array_equal(s1.cpu().numpy(), s2.cpu().numpy())


def test_fused_or_argument_errors():
    data = small(n=3000, d=32, nlist=4, sig_bits=64, B=4, nprobe=2, k=20, seed=100)
    g = data.to(torch.device("cuda"))
    idx = st.Index(g.items, g.sigs, g.offsets, g.centroids)
    try:
        too_many = torch.zeros((4, st.ST_MAX_OR + 1, 1), dtype=torch.int64, device="cuda")
        with pytest.raises(st.StError) as e:
            idx.search(g.queries, g.masks, 2, 20, or_masks=too_many)
        assert e.value.status == st.ST_ERR_INVALID_ARG
        host = torch.zeros((4, 2, 1), dtype=torch.int64)
        with pytest.raises(st.StError) as e:
            idx.search(g.queries, g.masks, 2, 20, or_masks=host)
        assert e.value.status == st.ST_ERR_INVALID_ARG
    finally:
        idx.close()
