"""GPU parity of the tensor-core (dense-unit) list scan: every case runs with
every probed list sent to the tensor cores (ST_OPT_DENSE_MIN_QUERIES = 1),
with none sent there (0) and at the default threshold, and each run must equal
the CPU oracle bit for bit (ids, int32 scores, probed lists, eligible counts).
The cases cover d = 64 and 128, 64- and 128-bit signatures, survivor densities
from a few per cent to nearly all rows, unions of mask bits wider than a unit's
plane slots (global planes), more than 32 queries on one list (several dense
units per chunk), ragged list tails, small k (the running top-k bound prunes
most keys) and k above the eligible count (nothing can be pruned)."""
import numpy as np
import pytest
import torch

import filtered_int8_ann_b200 as st
import oracle
from gpu_util import assert_parity, run_oracle
from workloads import WORKLOADS, generate, small, to_numpy

pytestmark = pytest.mark.gpu

CASES = [
    # nearly every row eligible, many queries per list
    dict(n=6000, d=128, nlist=4, sig_bits=128, hash_bits=3, B=40, nprobe=3, k=50, seed=101,
         mask_flags=1, mask_lang=False),
    dict(n=6000, d=64, nlist=4, sig_bits=128, hash_bits=3, B=40, nprobe=3, k=50, seed=102,
         mask_flags=1, mask_lang=False),
    dict(n=5000, d=128, nlist=5, sig_bits=64, hash_bits=2, B=24, nprobe=4, k=500, seed=103,
         mask_flags=0, mask_lang=False),
    dict(n=5000, d=64, nlist=5, sig_bits=64, hash_bits=2, B=24, nprobe=4, k=7, seed=104,
         mask_flags=0, mask_lang=False),
    # a few per cent eligible
    dict(n=9000, d=128, nlist=3, sig_bits=128, hash_bits=3, B=33, nprobe=2, k=100, seed=105, mask_flags=3),
    dict(n=9000, d=64, nlist=3, sig_bits=128, hash_bits=3, B=33, nprobe=2, k=100, seed=106, mask_flags=3),
    # item-mode masks: the unit's mask union exceeds the plane buffer (global planes)
    dict(n=8000, d=64, nlist=3, sig_bits=128, hash_bits=3, B=60, nprobe=3, k=150, seed=107,
         mask_mode="item", mask_country=True, mask_flags=2),
    # more than 32 queries per list: several dense units per chunk
    dict(n=7000, d=128, nlist=2, sig_bits=128, hash_bits=3, B=150, nprobe=2, k=64, seed=108,
         mask_flags=1, mask_lang=False),
    dict(n=7000, d=64, nlist=3, sig_bits=64, hash_bits=2, B=130, nprobe=2, k=300, seed=109, mask_flags=2),
    # k above the eligible count (no pruning possible), ragged lists, one query
    dict(n=3001, d=128, nlist=7, sig_bits=128, hash_bits=3, B=9, nprobe=7, k=4096, seed=110, mask_flags=2),
    dict(n=2500, d=64, nlist=6, sig_bits=64, B=1, nprobe=6, k=30, seed=111, mask_flags=1),
    # Zipf-skewed lists
    dict(n=30000, d=64, nlist=64, sig_bits=128, hash_bits=3, B=48, nprobe=16, k=200, seed=112,
         centroid_zipf=0.8, mask_flags=2),
    dict(n=30000, d=128, nlist=32, sig_bits=128, hash_bits=3, B=64, nprobe=8, k=1000, seed=113,
         centroid_zipf=0.8, mask_flags=1, mask_lang=False),
]


def _run(data, P, k, min_q, exclude=None, deleted=None):
    g = data.to(torch.device("cuda"))
    idx = st.Index(g.items, g.sigs, g.offsets, g.centroids)
    try:
        if min_q is not None:
            idx.set_option(st.ST_OPT_DENSE_MIN_QUERIES, min_q)
        if deleted is not None:
            idx.delete(torch.from_numpy(deleted).cuda())
        B = g.queries.shape[0]
        elig = torch.empty(B, dtype=torch.int64, device="cuda")
        cands = torch.empty(B, dtype=torch.int64, device="cuda")
        probe = torch.empty((B, P), dtype=torch.int32, device="cuda")
        ex = None if exclude is None else torch.from_numpy(exclude.view(np.int64)).cuda()
        ids, sc = idx.search(g.queries, g.masks, P, k, eligible=elig, probe=probe, candidates=cands, exclude=ex)
        assert idx.check() == st.ST_OK
        return (ids.cpu().numpy(), sc.cpu().numpy(), probe.cpu().numpy(), elig.cpu().numpy()), cands.cpu().numpy()
    finally:
        idx.close()


@pytest.mark.parametrize("case", CASES, ids=[f"case{i}" for i in range(len(CASES))])
def test_dense_scan_parity(case):
    data = small(**case)
    P, k = case["nprobe"], case["k"]
    exp = run_oracle(data, P, k)
    for min_q in (1, 0, None):
        got, cands = _run(data, P, k, min_q)
        assert_parity(got, exp, f"{case} dense_min_queries={min_q}")
        elig = got[3]
        assert np.all(cands <= elig), "more candidates written than eligible items"
        assert np.all(cands >= np.minimum(elig, k)), "fewer candidates than the top-k needs"


def test_dense_scan_prunes_candidates():
    # 40 queries over 64 lists of about 16k rows, 16 probed per query (one of
    # them the query's own cluster), nearly all rows eligible, k = 10, every
    # list on the tensor cores: once the first units have published a bound,
    # the keys of the other lists fall below it and are not written
    data = small(n=1_000_000, d=128, nlist=64, sig_bits=128, hash_bits=3, B=40, nprobe=16, k=10, seed=120,
                 mask_flags=1, mask_lang=False)
    exp = run_oracle(data, 16, 10)
    got, cands = _run(data, 16, 10, 1)
    assert_parity(got, exp, "pruned")
    assert cands.sum() < 0.8 * got[3].sum(), (cands.sum(), got[3].sum())


def test_dense_scan_with_deletions_and_exclude_masks():
    # post-filter inside the dense scan: deleted items and items matching a
    # query's exclude mask are neither written nor counted for the bound
    data = small(n=8000, d=64, nlist=4, sig_bits=128, hash_bits=3, B=36, nprobe=3, k=40, seed=121,
                 mask_flags=1, mask_lang=False)
    a = to_numpy(data)
    rng = np.random.default_rng(5)
    # delete the oracle's top results of the first queries plus random rows
    top = run_oracle(data, 3, 40)[0]
    deleted = np.unique(np.concatenate([top[:4, :20].ravel(), rng.choice(8000, 800, replace=False)]))
    deleted = deleted[deleted >= 0].astype(np.int64)
    x = np.zeros_like(a["masks"])
    x[::3] = a["sigs"][rng.choice(8000, x[::3].shape[0])] & np.uint64(0x0F0F0F0F0F0F0F0F)
    exp_i, exp_s = [], []
    for b in range(a["queries"].shape[0]):
        sg = a["sigs"].copy()
        sg[deleted] = 0
        if x[b].any():
            hit = np.all((a["sigs"] & x[b]) == x[b], axis=1)
            sg[hit] = 0
        r = oracle.search(a["items"], sg, a["offsets"], a["centroids"], a["queries"][b:b + 1],
                          a["masks"][b:b + 1], 3, 40)
        exp_i.append(r[0][0])
        exp_s.append(r[1][0])
    for min_q in (1, 0):
        got, _ = _run(data, 3, 40, min_q, exclude=x, deleted=deleted)
        assert np.array_equal(got[0], np.stack(exp_i)), f"ids differ (dense_min_queries={min_q})"
        assert np.array_equal(got[1], np.stack(exp_s)), f"scores differ (dense_min_queries={min_q})"


def test_dense_scan_sweep_batch():
    # the 10M batch-sweep workload at B = 1024: nearly every probed list has
    # eight or more queries, so the dense scan takes almost all units at the
    # default threshold; every query against the oracle, and the running bound
    # must keep most of the 127k eligible keys per query from being written
    wl = WORKLOADS["sweep_10m"]
    data = generate(wl.with_(B=1024), device="cuda")
    a = to_numpy(data)
    idx = st.Index(data.items, data.sigs, data.offsets, data.centroids)
    try:
        B = 1024
        cands = torch.empty(B, dtype=torch.int64, device="cuda")
        elig = torch.empty(B, dtype=torch.int64, device="cuda")
        ids, sc = idx.search(data.queries, data.masks, wl.nprobe, wl.k, eligible=elig, candidates=cands)
        assert idx.check() == st.ST_OK
        r = oracle.search(a["items"], a["sigs"], a["offsets"], a["centroids"], a["queries"], a["masks"],
                          wl.nprobe, wl.k, nthreads=oracle.max_threads())
        assert np.array_equal(ids.cpu().numpy(), r[0])
        assert np.array_equal(sc.cpu().numpy(), r[1])
        assert np.array_equal(elig.cpu().numpy(), r[3])
        assert float(cands.sum()) < 0.25 * float(elig.sum()), (float(cands.sum()), float(elig.sum()))
    finally:
        idx.close()


def test_dense_bound_ignores_deleted_keys_of_the_warp_scan():
    # one query (X) probes a list of 600 rows that no other query probes (the
    # warp scan takes it) and a 1M-row list shared with eight other queries
    # (the tensor cores take it). Every row of the small list is deleted and
    # scores far above anything live for X; X's best live rows are the last
    # rows of the large list, which the dense scan reaches after its first
    # units have raised X's running bound. That bound must count only keys
    # that can be results: the warp scan leaves deleted items to the final
    # top-k's post-filter, so it must not count them in the score bins the
    # dense scan reads, or X's true results are pruned.
    rng = np.random.default_rng(141)
    nA, nB, nC, d = 1_000_000, 600, 4096, 64
    n = nA + nB + nC
    items = rng.integers(-20, 21, size=(n, d)).astype(np.int8)
    items[:nA, 0] += 40
    items[nA - 2048:nA, 1] = 40
    items[nA:nA + nB, 1] = 100
    items[nA + nB:, 2] += 40
    sigs = np.ones((n, 1), dtype=np.uint64)
    offsets = np.array([0, nA, nA + nB, n], dtype=np.int64)
    cent = np.zeros((3, d), dtype=np.int8)
    cent[0, 0] = cent[1, 1] = cent[2, 2] = 100
    q = np.zeros((9, d), dtype=np.int8)
    q[:8, 0] = 40
    q[:8, 2] = 40
    q[:8, 3:] = rng.integers(-3, 4, size=(8, d - 3))
    q[8, 0], q[8, 1] = 30, 60
    masks = np.ones((9, 1), dtype=np.uint64)
    deleted = np.arange(nA, nA + nB, dtype=np.int64)
    live = sigs.copy()
    live[deleted] = 0
    P, k = 2, 20
    exp = oracle.search(items, live, offsets, cent, q, masks, P, k, nthreads=oracle.max_threads())
    assert exp[2][8].tolist() == [1, 0] and all(r == [0, 2] for r in exp[2][:8].tolist())
    dev = lambda x, dt: torch.from_numpy(np.ascontiguousarray(x).view(dt)).cuda()
    idx = st.Index(dev(items, np.int8), dev(sigs, np.int64), dev(offsets, np.int64), dev(cent, np.int8))
    try:
        idx.delete(torch.from_numpy(deleted).cuda())
        ids, sc = idx.search(dev(q, np.int8), dev(masks, np.int64), P, k)
        assert idx.check() == st.ST_OK
        assert np.array_equal(sc.cpu().numpy(), exp[1]), (sc.cpu().numpy()[8][:4], exp[1][8][:4])
        assert np.array_equal(ids.cpu().numpy(), exp[0])
    finally:
        idx.close()


def test_selectivity_routes_small_lists_to_the_tensor_cores():
    # 512 lists of ~3.9k rows, 64 queries x 32 probes (2048 probes): lists
    # are probed by ~4 queries, below the default threshold of 8, but one-flag
    # masks pass ~90 % of the rows, so the queries' sampled selectivities send
    # their lists to the tensor cores. The warp scan writes every eligible key,
    # the dense scan only keys that can still reach the top-k: fewer candidates
    # than eligible items show which scan ran. Results equal the oracle's.
    data = small(n=2_000_000, d=128, nlist=512, sig_bits=128, hash_bits=3, B=64, nprobe=32, k=100, seed=151,
                 mask_flags=1, mask_lang=False)
    exp = run_oracle(data, 32, 100)
    got, cands = _run(data, 32, 100, None)
    assert_parity(got, exp, "selectivity-routed")
    per_list = np.bincount(got[2].ravel(), minlength=512)
    assert np.median(per_list[per_list > 0]) < 8, per_list
    assert cands.sum() < 0.5 * got[3].sum(), (cands.sum(), got[3].sum())
    got0, cands0 = _run(data, 32, 100, 0)  # tensor cores off: every eligible key written
    assert_parity(got0, exp, "warp scan only")
    assert np.array_equal(cands0, got0[3])
