// Final top-k for k <= ST_SMALL_K: one thread-block cluster per query
// (cluster_topk.cuh).
//
// Same result as the chunked kernels of select.cu (the k best candidate keys
// of each query, score descending then item id ascending, padded with id -1 /
// INT32_MIN) -- SilverTorch: Index as Model, section on redesigning each
// stage as a pure PyTorch module, fused Int8 ANN paragraph (a large result
// pool); maximum top-k row of the compute cost efficiency table in the
// Spanish translation -- in one launch and without global atomics: the CS
// CTAs of a query's cluster split its candidates and talk through distributed
// shared memory.
//   1. each CTA histograms its share of the keys (2048 bins over the query's
//      score range, which the scan recorded) in its own shared memory;
//   2. the leader (rank 0) sums the CS histograms through DSMEM and finds the
//      cut bin (the one holding the k-th best key) and every higher bin's
//      output segment;
//   3. every CTA reads its share again and sends each key above the cut
//      straight to its segment in the leader's shared memory (DSMEM atomics
//      on the segment cursors), and each key of the cut bin to the leader's
//      tie buffer;
//   4. the leader takes the cut bin's best, ranks every segment and writes the
//      ids and scores.
// A query whose candidates overflowed the scan's buffer takes the exact
// overflow path in the leader alone (the other CTAs of its cluster return at
// once, before any cluster barrier, so no barrier waits for them).
#include "cluster_topk.cuh"
#include "select_common.cuh"

namespace cg = cooperative_groups;

namespace st {

constexpr int kCBlock = 512;
constexpr int kCTieCap = 4096;

template <int CS>
__global__ void __launch_bounds__(kCBlock)
select_cluster_kernel(SearchArgs a)
{
    dep_enter();
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = int(cluster.block_rank());
    const int q = int(blockIdx.x) / CS;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ SelectSmem ss;
    __shared__ ClusterCut cc;
    const int k = a.k;
    const int pwk = next_pow2(k);
    // shared layout: [tmp: k keys, rounded up to even][tie: kCTieCap keys][out: next_pow2(k) keys]
    uint64_t* tmp = reinterpret_cast<uint64_t*>(smem_raw);
    uint64_t* tie = tmp + ((k + 1) & ~1);
    uint64_t* out = tie + kCTieCap;
    const int tid = threadIdx.x;

    const uint32_t cnt = a.cand_cnt[int64_t(q) * kCntStride];
    const int64_t n = cnt;
    uint64_t* keys = a.cand + int64_t(q) * a.cap;
    const bool filt = a.dead || a.qexclude;
    int m = 0;

    if (n > a.cap || n == 0) {
        // (cluster-uniform) the scan overflowed this query's buffer, or no
        // candidate: the leader alone, and no cluster barrier
        if (rank != 0) return;
        if (n > 0) {
            const int64_t nk = overflow_path<kCBlock>(a, q, out, pwk, reinterpret_cast<int4*>(tie), ss);
            // the kept keys are at the front of the candidate buffer
            m = block_topk_sorted<kCBlock>(keys, nk, k, out, tmp, tie, kCTieCap, false, 0, 0, ss, a.err);
        }
    } else {
        // the scan recorded a range containing every candidate's score
        const uint32_t* qr = a.score_rng + int64_t(q) * kCntStride;
        const int32_t hi = int32_t(qr[0] ^ 0x80000000u);
        const int32_t lo = int32_t(~qr[1] ^ 0x80000000u);
        auto keep = [&](uint64_t key) { return keep_item(a, q, key_id(key)); };
        auto compact = [&]() { return compact_cut_bin<kCBlock>(a, q, n, cc.t); };
        m = cluster_topk<CS, kCBlock>(cluster, keys, n, k, true, lo, hi, filt, keep, compact, tmp, tie, kCTieCap,
                                      out, ss, cc, a.err);
        if (m < 0) return;  // not the leader
    }
    for (int r = tid; r < k; r += kCBlock) {
        const uint64_t key = r < m ? out[r] : 0ull;  // key 0 reads as (id -1, INT32_MIN)
        a.out_ids[int64_t(q) * k + r] = key == 0ull ? -1 : key_id(key) + a.id_offset;
        a.out_scores[int64_t(q) * k + r] = key_score(key);
    }
    if (tid == 0 && a.out_eligible) a.out_eligible[q] = int64_t(a.eligible_cnt[int64_t(q) * (kCntStride / 2)]);
    if (tid == 0 && a.out_cands) a.out_cands[q] = int64_t(cnt);
}

size_t select_cluster_smem(int k)
{
    return (size_t((k + 1) & ~1) + kCTieCap + size_t(next_pow2(k))) * 8;
}

template <int CS>
static cudaError_t launch_cs(const SearchArgs& a, cudaStream_t s)
{
    const size_t smem = select_cluster_smem(ST_SMALL_K);  // the attribute covers every k
    const void* fn = reinterpret_cast<const void*>(select_cluster_kernel<CS>);
    cudaError_t e = ensure_smem_attr(fn, int(smem));
    if (e != cudaSuccess) return e;
    return launch_dep_cluster(select_cluster_kernel<CS>, dim3(unsigned(a.B) * CS), dim3(kCBlock),
                              select_cluster_smem(a.k), CS, s, a);
}

cudaError_t launch_select_cluster(const SearchArgs& a, int num_sms, cudaStream_t s)
{
    switch (cluster_size_for(a.B, num_sms)) {
    case 8: return launch_cs<8>(a, s);
    case 4: return launch_cs<4>(a, s);
    case 2: return launch_cs<2>(a, s);
    default: return launch_cs<1>(a, s);
    }
}

}  // namespace st
