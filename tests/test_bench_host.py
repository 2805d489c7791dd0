"""Host-side statistics of the benchmark on CPU tensors: the Bloom
false-positive count it reports, against an independent numpy count over the
same probed lists (the oracle's probe) and the generator's exact attributes."""
import numpy as np
import torch

import bench
import bruteforce as bf
import oracle
from workloads import small, to_numpy


def _numpy_fp(data, a, lists_per_query):
    lang, country, flags = data.lang.numpy(), data.country.numpy(), data.flags.numpy()
    passed = fp = fn = 0
    for b, lists in enumerate(lists_per_query):
        rows = np.concatenate([np.arange(a["offsets"][c], a["offsets"][c + 1]) for c in lists])
        ok = bf.bloom_pass(a["sigs"][rows], a["masks"][b])
        exact = np.ones(rows.size, bool)
        if int(data.q_lang[b]) >= 0:
            exact &= lang[rows] == int(data.q_lang[b])
        if int(data.q_country[b]) >= 0:
            exact &= country[rows] == int(data.q_country[b])
        for f in np.nonzero(data.q_flags[b].numpy())[0]:
            exact &= flags[rows, f]
        passed += int(ok.sum())
        fp += int((ok & ~exact).sum())
        fn += int((exact & ~ok).sum())
    return passed, fp, fn


def test_bloom_false_positive_count_matches_numpy():
    for kw in (dict(n=6000, d=32, nlist=12, sig_bits=64, hash_bits=3, B=10, nprobe=4, k=50, seed=5,
                    mask_country=True, mask_flags=2),
               dict(n=5000, d=32, nlist=8, sig_bits=128, hash_bits=2, B=6, nprobe=3, k=50, seed=6,
                    mask_mode="item", mask_country=True, mask_flags=1)):
        data = small(**kw)
        a = to_numpy(data)
        lists = [oracle.probe(a["queries"][b], a["centroids"], kw["nprobe"]) for b in range(kw["B"])]
        probe = torch.from_numpy(np.stack(lists))
        got = bench.bloom_fp(data, probe, 0)
        exp = _numpy_fp(data, a, lists)
        assert got == exp
        assert got[2] == 0  # no false negatives
    # the 64-bit case has collisions: some false positives are expected
    data = small(n=6000, d=32, nlist=12, sig_bits=64, hash_bits=3, B=10, nprobe=4, k=50, seed=5,
                 mask_country=True, mask_flags=2)
    a = to_numpy(data)
    lists = [oracle.probe(a["queries"][b], a["centroids"], 4) for b in range(10)]
    assert bench.bloom_fp(data, torch.from_numpy(np.stack(lists)), 0)[1] > 0


def test_bloom_false_positive_count_uses_the_batch_rows():
    """Batch b of the pool is rows q0 .. q0+B-1 of the generated queries."""
    data = small(n=4000, d=32, nlist=8, sig_bits=64, hash_bits=3, B=12, nprobe=3, k=20, seed=7,
                 mask_country=True, mask_flags=2)
    a = to_numpy(data)
    lists = [oracle.probe(a["queries"][b], a["centroids"], 3) for b in range(12)]
    probe = torch.from_numpy(np.stack(lists))
    whole = bench.bloom_fp(data, probe, 0)
    halves = [bench.bloom_fp(data, probe[h * 6:(h + 1) * 6], h * 6) for h in range(2)]
    assert tuple(x + y for x, y in zip(*halves)) == whole


def test_cpu_baseline_reports_parallel_and_single_thread_rates():
    data = small(n=3000, d=32, nlist=8, sig_bits=64, B=8, nprobe=3, k=20, seed=9)
    q = data.queries.reshape(2, 4, -1)
    m = data.masks.reshape(2, 4, -1)
    wl = data.wl.with_(B=4)
    cpu = bench.cpu_baseline(data, q, m, wl, 0.3)
    assert cpu["kind"] == "oracle" and cpu["unit"] == "queries/s" and cpu["value"] > 0
    assert cpu["cores"] == oracle.max_threads()
    assert cpu["single_thread"]["value"] > 0 and cpu["single_thread"]["unit"] == "queries/s"
    assert "cpu_model" in cpu


class _Peaks:
    hbm_gbs = 1000.0          # 1 ms per GB
    int8_tensor_tops = 1000.0  # 1 ms per 10^12 ops
    dp4a_tops = 100.0          # 10 ms per 10^12 ops


def test_roofline_splits_the_int8_products_between_tensor_cores_and_dp4a():
    # 1 GB and 10^12 products measured in 20 ms: HBM 1 ms; compute 10 ms on
    # dp4a alone, 1 ms on the tensor cores alone, 0.5 + 5 ms half and half
    r = bench.roofline(1e9, 1e12, 20.0, _Peaks, 0.0)
    assert r["bound"] == "alu" and abs(r["frac"] - 0.5) < 1e-12 and abs(r["hbm_frac"] - 0.05) < 1e-12
    r = bench.roofline(1e9, 1e12, 20.0, _Peaks, 1.0)
    assert r["bound"] == "hbm" and abs(r["frac"] - 0.05) < 1e-12 and abs(r["compute_frac"] - 0.05) < 1e-12
    r = bench.roofline(1e9, 1e12, 20.0, _Peaks, 0.5)
    assert r["bound"] == "alu" and abs(r["compute_frac"] - 5.5 / 20.0) < 1e-12
    r = bench.roofline(1e8, 4e12, 20.0, _Peaks, 1.0)
    assert r["bound"] == "tensor" and abs(r["frac"] - 0.2) < 1e-12


def test_byte_model_counts_dense_list_pairs():
    # every query probes every list: with the threshold at B all pairs are in
    # dense lists (d = 64 has the tensor-core scan), with 0 none are
    data = small(n=3000, d=64, nlist=4, sig_bits=64, B=9, nprobe=4, k=20, seed=11, mask_flags=1)
    probe = torch.arange(4, dtype=torch.int32).repeat(9, 1)
    old = bench.DENSE_MIN_Q
    try:
        bench.DENSE_MIN_Q = 9
        assert bench.byte_model(data, probe, data.masks, 1, 64, 20, 4)["dense_pair_frac"] == 1.0
        bench.DENSE_MIN_Q = 10
        assert bench.byte_model(data, probe, data.masks, 1, 64, 20, 4)["dense_pair_frac"] == 0.0
        bench.DENSE_MIN_Q = 0
        assert bench.byte_model(data, probe, data.masks, 1, 64, 20, 4)["dense_pair_frac"] == 0.0
    finally:
        bench.DENSE_MIN_Q = old
