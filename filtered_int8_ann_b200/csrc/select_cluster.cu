// Final top-k for k <= ST_SMALL_K: one thread-block cluster per query.
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
#include <cooperative_groups.h>

#include "select_common.cuh"

namespace cg = cooperative_groups;

namespace st {

constexpr int kCBlock = 512;
constexpr int kCTieCap = 4096;

struct ClusterCut {
    TopkCut t;
    uint32_t tpos;  // cut-bin keys sent to the leader
};

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
    // leader's shared layout: [tmp: k keys, rounded up to even][tie: kCTieCap keys][out: next_pow2(k) keys]
    uint64_t* tmp = reinterpret_cast<uint64_t*>(smem_raw);
    uint64_t* tie = tmp + ((k + 1) & ~1);
    uint64_t* out = tie + kCTieCap;
    const int tid = threadIdx.x;

    const uint32_t cnt = a.cand_cnt[int64_t(q) * kCntStride];
    const int64_t n = cnt;
    const uint64_t* keys = a.cand + int64_t(q) * a.cap;
    const bool filt = a.dead || a.qexclude;
    int m = 0;

    if (n > a.cap || n == 0) {
        // (cluster-uniform) the scan overflowed this query's buffer, or no
        // candidate: the leader alone
        if (rank != 0) return;
        if (n > 0) {
            const int64_t nk = overflow_path<kCBlock>(a, q, out, pwk, reinterpret_cast<int4*>(tie), ss);
            // the kept keys are at the front of the candidate buffer
            m = block_topk_sorted<kCBlock>(keys, nk, k, out, tmp, tie, kCTieCap, false, 0, 0, ss, a.err);
        }
    } else {
        int32_t lo;
        uint32_t sh;
        query_range(a, q, lo, sh);
        const int64_t s0 = n * rank / CS, s1 = n * (rank + 1) / CS;
        // 1. this CTA's histogram
        for (int i = tid; i < kSelBins; i += kCBlock) ss.hist[i] = 0;
        if (rank == 0 && tid == 0) cc.tpos = 0;
        __syncthreads();
        constexpr int U = 8;
        for (int64_t base = s0; base < s1; base += int64_t(kCBlock) * U) {
            uint64_t v[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t i = base + int64_t(u) * kCBlock + tid;
                v[u] = i < s1 ? keys[i] : 0ull;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t i = base + int64_t(u) * kCBlock + tid;
                if (i < s1 && (!filt || keep_item(a, q, key_id(v[u])))) atomicAdd(&ss.hist[topk_bin(v[u], lo, sh)], 1u);
            }
        }
        cluster.sync();  // every CTA's histogram is complete
        // 2. the leader sums them and finds the cut
        if (rank == 0) {
            uint32_t local = 0;
            for (int i = tid; i < kSelBins; i += kCBlock) {
                uint32_t tot = ss.hist[i];
#pragma unroll 1
                for (int r = 1; r < CS; ++r) tot += cluster.map_shared_rank(&ss.hist[0], r)[i];
                ss.hist[i] = tot;
                local += tot;
            }
            uint32_t nk;
            block_excl_scan<kCBlock>(local, ss.part, nk);
            const TopkCut t = topk_cut_from_hist<kCBlock>(int64_t(nk), k, lo, sh, ss);
            if (tid == 0) cc.t = t;
        }
        cluster.sync();  // the cut and the leader's segment cursors are ready
        // 3. keys above the cut to their segments, cut-bin keys to the tie buffer
        {
            ClusterCut* lc = cluster.map_shared_rank(&cc, 0);
            const int cut = lc->t.cut;
            uint32_t* cursor = cluster.map_shared_rank(&ss.hist[0], 0);
            uint32_t* tpos = &lc->tpos;
            uint64_t* ltmp = cluster.map_shared_rank(tmp, 0);
            uint64_t* ltie = cluster.map_shared_rank(tie, 0);
            for (int64_t base = s0; base < s1; base += int64_t(kCBlock) * U) {
                uint64_t v[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int64_t i = base + int64_t(u) * kCBlock + tid;
                    v[u] = i < s1 ? keys[i] : 0ull;
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int64_t i = base + int64_t(u) * kCBlock + tid;
                    if (i >= s1) continue;
                    const int b = topk_bin(v[u], lo, sh);
                    if (b < cut) continue;
                    if (filt && !keep_item(a, q, key_id(v[u]))) continue;
                    if (b > cut) {
                        ltmp[atomicAdd(&cursor[b], 1u)] = v[u];
                    } else {
                        const uint32_t tp = atomicAdd(tpos, 1u);
                        if (tp < uint32_t(kCTieCap)) ltie[tp] = v[u];
                    }
                }
            }
        }
        cluster.sync();  // every key is in the leader's memory
        if (rank != 0) return;
        // 4. the leader: the cut bin's best, then every segment's order
        TopkCut t = cc.t;
        const uint64_t* tsrc = tie;
        if (t.tcount > kCTieCap) {
            tsrc = nullptr;  // select over all keys of the cut bin in global memory
            if (filt && t.m > t.above) {
                const int nt = compact_cut_bin<kCBlock>(a, q, n, t);
                t.tcount = nt;
                tsrc = keys;
            }
        }
        topk_take_ties<kCBlock>(t, tsrc, keys, n, tmp, ss, a.err);
        topk_rank<kCBlock>(t, tmp, out, ss);
        m = t.m;
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
    cudaError_t e = ensure_smem_attr(fn, 24 + (CS == 1 ? 0 : CS == 2 ? 1 : CS == 4 ? 2 : 3), int(smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(a.B) * CS);
    cfg.blockDim = dim3(kCBlock);
    cfg.dynamicSmemBytes = select_cluster_smem(a.k);
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = CS;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, select_cluster_kernel<CS>, a);
}

// CTAs per query: enough clusters to cover the SMs at small batches.
int select_cluster_size(int B, int num_sms)
{
    if (B * 8 <= 2 * num_sms) return 8;
    if (B * 4 <= 2 * num_sms) return 4;
    if (B * 2 <= 2 * num_sms) return 2;
    return 1;
}

cudaError_t launch_select_cluster(const SearchArgs& a, int num_sms, cudaStream_t s)
{
    switch (select_cluster_size(a.B, num_sms)) {
    case 8: return launch_cs<8>(a, s);
    case 4: return launch_cs<4>(a, s);
    case 2: return launch_cs<2>(a, s);
    default: return launch_cs<1>(a, s);
    }
}

}  // namespace st
