"""GPU parity: the CUDA path against the CPU oracle, element by element and bit
exact (ids, int32 scores, probed lists, eligible counts), on seeded inputs
spanning several work units and ragged tails, every code path of the scan
(d held in registers or not, 64- and 128-bit signatures, more than 32 queries
per list) and the degenerate cases of the method."""
import numpy as np
import pytest
import torch

import filtered_int8_ann_b200 as st
from gpu_util import assert_parity, run_gpu, run_oracle
from workloads import WORKLOADS, generate, small

pytestmark = pytest.mark.gpu

CASES = [
    dict(n=3000, d=64, nlist=16, sig_bits=128, hash_bits=3, B=8, nprobe=4, k=50, seed=1),
    dict(n=5000, d=128, nlist=12, sig_bits=128, hash_bits=3, B=16, nprobe=5, k=300, seed=2),
    dict(n=4000, d=64, nlist=20, sig_bits=64, B=8, nprobe=6, k=64, seed=3),
    dict(n=4000, d=128, nlist=9, sig_bits=64, B=5, nprobe=9, k=1000, seed=4),
    dict(n=2500, d=16, nlist=7, sig_bits=64, B=6, nprobe=3, k=40, seed=5),
    dict(n=2500, d=48, nlist=7, sig_bits=128, B=6, nprobe=3, k=40, seed=6),
    dict(n=2000, d=512, nlist=5, sig_bits=128, B=4, nprobe=2, k=33, seed=7),
    dict(n=2000, d=96, nlist=5, sig_bits=64, B=4, nprobe=5, k=77, seed=8),
    # more than 32 queries probing the same lists (several query groups per unit)
    dict(n=6000, d=64, nlist=4, sig_bits=128, B=100, nprobe=2, k=128, seed=9, mask_flags=1),
    dict(n=6000, d=128, nlist=3, sig_bits=64, B=70, nprobe=3, k=200, seed=10, mask_flags=0, mask_lang=False),
    # Zipf-skewed lists, item-mode masks
    dict(n=20000, d=64, nlist=64, sig_bits=128, hash_bits=3, B=24, nprobe=8, k=256, seed=11,
         centroid_zipf=0.8, mask_mode="item", mask_country=True),
    # flat uniform
    dict(n=30000, d=128, nlist=1, sig_bits=128, hash_bits=3, B=2, nprobe=1, k=2048, seed=12,
         uniform_items=True, mask_flags=2),
    # item-mode masks (language and country vary per query) and many queries per
    # list: a unit's mask union exceeds the 32-plane buffer, so the scan tests
    # from the global planes
    dict(n=8000, d=64, nlist=3, sig_bits=128, hash_bits=3, B=60, nprobe=3, k=150, seed=15,
         mask_mode="item", mask_country=True, mask_flags=2),
    dict(n=8000, d=128, nlist=2, sig_bits=64, hash_bits=2, B=40, nprobe=2, k=90, seed=16,
         mask_mode="item", mask_country=True, mask_flags=3),
    # k = 1 and k = 4096
    dict(n=9000, d=64, nlist=10, sig_bits=64, B=3, nprobe=10, k=1, seed=13),
    dict(n=9000, d=64, nlist=10, sig_bits=128, B=3, nprobe=10, k=4096, seed=14, mask_flags=0,
         mask_lang=False),
]


@pytest.mark.parametrize("case", CASES, ids=[f"case{i}" for i in range(len(CASES))])
def test_parity_small(case):
    data = small(**case)
    P, k = case["nprobe"], case["k"]
    assert_parity(run_gpu(data, P, k), run_oracle(data, P, k), str(case))


def test_parity_tiny_ivf_and_flat():
    data = generate(WORKLOADS["tiny_ivf"])
    wl = data.wl
    assert_parity(run_gpu(data, wl.nprobe, wl.k), run_oracle(data, wl.nprobe, wl.k), "tiny_ivf")
    f = data.flat()
    assert_parity(run_gpu(f, 1, wl.k), run_oracle(f, 1, wl.k), "tiny_flat")
    # IVF with nprobe = nlist equals flat
    a = run_gpu(data, wl.nlist, wl.k)
    b = run_gpu(f, 1, wl.k)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    # item-mode masks
    d2 = generate(WORKLOADS["tiny_ivf"], mask_mode="item")
    assert_parity(run_gpu(d2, wl.nprobe, wl.k), run_oracle(d2, wl.nprobe, wl.k), "tiny_ivf item")


def test_parity_mid_ivf():
    data = generate(WORKLOADS["mid_ivf"])
    wl = data.wl
    assert_parity(run_gpu(data, wl.nprobe, wl.k), run_oracle(data, wl.nprobe, wl.k), "mid_ivf")


def test_wide_mask_union_uses_global_planes():
    """The unit-level union of 60 item-mode masks has more than 32 bits."""
    data = small(n=8000, d=64, nlist=3, sig_bits=128, hash_bits=3, B=60, nprobe=3, k=150, seed=15,
                 mask_mode="item", mask_country=True, mask_flags=2)
    m = data.masks.numpy().view(np.uint64)
    union = np.bitwise_or.reduce(m[:32], axis=0)
    assert sum(bin(int(w)).count("1") for w in union) > 32
    assert_parity(run_gpu(data, 3, 150), run_oracle(data, 3, 150), "wide union")


def test_padding_when_few_eligible():
    data = small(n=3000, d=64, nlist=8, B=4, nprobe=2, k=3000, seed=21, mask_flags=6,
                 mask_country=True)
    got = run_gpu(data, 2, 3000)
    assert_parity(got, run_oracle(data, 2, 3000), "padding")
    assert (got[0] == -1).any() and (got[1] == np.iinfo(np.int32).min).any()


def test_mask_zero_and_all_ones():
    data = small(n=3000, d=64, nlist=8, B=4, nprobe=3, k=100, seed=22)
    data.masks.zero_()
    assert_parity(run_gpu(data, 3, 100), run_oracle(data, 3, 100), "mask 0")
    data.masks.fill_(-1)  # all ones: only all-ones signatures pass
    data.sigs[::97] = -1
    assert_parity(run_gpu(data, 3, 100), run_oracle(data, 3, 100), "mask all ones")


def test_extreme_int8_values():
    data = small(n=4000, d=128, nlist=6, B=4, nprobe=6, k=500, seed=23)
    data.items[::3] = 127
    data.items[1::3] = -128
    data.queries[0] = -128
    data.queries[1] = 127
    data.centroids[0] = -128
    assert_parity(run_gpu(data, 6, 500), run_oracle(data, 6, 500), "extremes")


def test_empty_lists_and_identical_items():
    data = small(n=2000, d=32, nlist=12, B=5, nprobe=12, k=700, seed=24)
    # make lists 0, 3 and 11 empty by moving their boundaries
    off = data.offsets.clone()
    off[1] = off[0]
    off[4] = off[3]
    off[11] = off[12]
    data.offsets = off
    data.items[:] = data.items[0]
    assert_parity(run_gpu(data, 12, 700), run_oracle(data, 12, 700), "empty lists")


def test_overflow_path_is_exact():
    # a candidate capacity far below the eligible count forces the exact
    # per-query fallback
    data = small(n=20000, d=64, nlist=4, sig_bits=128, B=6, nprobe=4, k=200, seed=25, mask_flags=0,
                 mask_lang=False)
    exp = run_oracle(data, 4, 200)
    assert exp[3].min() > 1300
    assert_parity(run_gpu(data, 4, 200, cap=200 + 1024), exp, "overflow")
    data2 = small(n=20000, d=128, nlist=3, sig_bits=64, B=3, nprobe=3, k=4096, seed=26, mask_flags=0,
                  mask_lang=False)
    assert_parity(run_gpu(data2, 3, 4096, cap=1), run_oracle(data2, 3, 4096), "overflow k=4096")


def test_deterministic_repeats_and_shared_index():
    data = small(n=8000, d=64, nlist=16, B=12, nprobe=5, k=200, seed=27).to("cuda")
    idx = st.Index(data.items, data.sigs, data.offsets, data.centroids)
    try:
        s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
        r1 = run_gpu(data, 5, 200, index=idx, stream=s1)
        r2 = run_gpu(data, 5, 200, index=idx, stream=s2)
        for x, y in zip(r1, r2):
            assert np.array_equal(x, y)
        assert_parity(r1, run_oracle(data.to("cpu"), 5, 200), "repeat")
    finally:
        idx.close()


def test_search_host_matches_device_path():
    data = small(n=8000, d=128, nlist=16, sig_bits=128, B=9, nprobe=4, k=150, seed=28)
    g = data.to("cuda")
    idx = st.Index(g.items, g.sigs, g.offsets, g.centroids)
    try:
        q = data.queries.pin_memory()
        m = data.masks.pin_memory()
        ids, sc = idx.search_host(q, m, 4, 150)
        exp = run_oracle(data, 4, 150)
        assert np.array_equal(ids.numpy(), exp[0]) and np.array_equal(sc.numpy(), exp[1])
        ids2, sc2 = idx.search_host(data.queries, data.masks, 4, 150)  # pageable memory
        assert torch.equal(ids, ids2) and torch.equal(sc, sc2)
    finally:
        idx.close()


def test_search_host_async_pipelined_matches_oracle():
    """Two batches in flight on two streams through the asynchronous host call,
    each slot's outputs checked when its stream is done; pageable buffers are
    refused before anything is enqueued."""
    data = small(n=12000, d=64, nlist=24, sig_bits=128, hash_bits=3, B=24, nprobe=6, k=300, seed=31)
    g = data.to("cuda")
    exp = run_oracle(data, 6, 300)
    idx = st.Index(g.items, g.sigs, g.offsets, g.centroids)
    try:
        halves = [(0, 12), (12, 24)]
        qs = [data.queries[a:b].contiguous().pin_memory() for a, b in halves]
        ms = [data.masks[a:b].contiguous().pin_memory() for a, b in halves]
        streams = [torch.cuda.Stream(), torch.cuda.Stream()]
        outs = [(torch.full((12, 300), -7, dtype=torch.int64).pin_memory(),
                 torch.full((12, 300), -7, dtype=torch.int32).pin_memory()) for _ in range(2)]
        for rep in range(3):
            for j in range(2):
                idx.search_host_async(qs[j], ms[j], 6, 300, outs[j][0], outs[j][1], stream=streams[j])
            for j, (a, b) in enumerate(halves):
                streams[j].synchronize()
                assert np.array_equal(outs[j][0].numpy(), exp[0][a:b])
                assert np.array_equal(outs[j][1].numpy(), exp[1][a:b])
                outs[j][0].fill_(-7)
        assert idx.check() == st.ST_OK
        pageable = torch.empty((12, 300), dtype=torch.int64)
        with pytest.raises(st.StError) as ei:
            idx.search_host_async(qs[0], ms[0], 6, 300, pageable, outs[0][1])
        assert ei.value.status == st.ST_ERR_INVALID_ARG
        with pytest.raises(st.StError) as ei:
            idx.search_host_async(data.queries[:12].contiguous(), ms[0], 6, 300, outs[0][0], outs[0][1])
        assert ei.value.status == st.ST_ERR_INVALID_ARG
        assert bool((outs[0][0] == -7).all())
    finally:
        idx.close()


def test_index_independent_of_caller_buffers():
    data = small(n=5000, d=64, nlist=8, B=4, nprobe=3, k=80, seed=29)
    g = data.to("cuda")
    idx = st.Index(g.items, g.sigs, g.offsets, g.centroids)
    try:
        g.items.zero_()
        g.sigs.zero_()
        q, m = data.queries.cuda(), data.masks.cuda()
        ids, sc = idx.search(q, m, 3, 80)
        exp = run_oracle(data, 3, 80)
        assert np.array_equal(ids.cpu().numpy(), exp[0]) and np.array_equal(sc.cpu().numpy(), exp[1])
    finally:
        idx.close()


def test_host_side_errors_with_device_buffers():
    data = small(n=2000, d=64, nlist=8, B=4, nprobe=3, k=10, seed=30).to("cuda")
    idx = st.Index(data.items, data.sigs, data.offsets, data.centroids)
    h = idx.handle
    L = st.lib()
    ids = torch.empty((4, 10), dtype=torch.int64, device="cuda")
    sc = torch.empty((4, 10), dtype=torch.int32, device="cuda")
    q, m = data.queries, data.masks
    s = torch.cuda.current_stream().cuda_stream
    try:
        call = lambda B=4, P=3, k=10, qp=q.data_ptr(), mp=m.data_ptr(), ip=ids.data_ptr(), sp=sc.data_ptr(): \
            L.st_search(h, qp, mp, B, P, k, ip, sp, s)
        assert call() == st.ST_OK
        assert call(B=0) == st.ST_ERR_INVALID_ARG
        assert call(k=0) == st.ST_ERR_INVALID_ARG
        assert call(P=0) == st.ST_ERR_INVALID_ARG
        assert call(P=9) == st.ST_ERR_INVALID_ARG          # nprobe > nlist
        assert call(k=st.ST_MAX_K + 1) == st.ST_ERR_UNSUPPORTED
        assert call(B=st.ST_MAX_B + 1) == st.ST_ERR_UNSUPPORTED   # checked before any buffer is read
        host = torch.empty((4, 64), dtype=torch.int8)
        assert call(qp=host.data_ptr()) == st.ST_ERR_INVALID_ARG   # host pointer
        assert call(qp=q.data_ptr() + 1) == st.ST_ERR_INVALID_ARG  # misaligned
        assert call(ip=0) == st.ST_ERR_INVALID_ARG
        # malformed offsets
        bad = data.offsets.clone()
        bad[3] = bad[4] + 1
        with pytest.raises(st.StError) as ei:
            st.Index(data.items, data.sigs, bad, data.centroids)
        assert ei.value.status == st.ST_ERR_INVALID_ARG
        bad = data.offsets.clone()
        bad[-1] -= 1
        with pytest.raises(st.StError):
            st.Index(data.items, data.sigs, bad, data.centroids)
        assert idx.check() == st.ST_OK
    finally:
        idx.close()
