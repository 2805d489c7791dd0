// Top-k of one key array by a thread-block cluster: the CS CTAs of the cluster
// split the keys, and the leader (rank 0) ends up with the k best, sorted
// descending. Used by the coarse probe (a query's nprobe best lists) and the
// final top-k (a query's k best candidates).
//   0. unless the caller knows it, the keys' score range: each CTA's min and
//      max, exchanged through distributed shared memory (DSMEM);
//   1. each CTA histograms its share of the keys (kSelBins bins over the
//      range) in its own shared memory;
//   2. the leader sums the CS histograms through DSMEM and finds the cut bin
//      (the one holding the k-th best key) and each higher bin's output
//      segment;
//   3. every CTA reads its share again and sends each key above the cut to its
//      segment in the leader's shared memory (DSMEM atomics on the leader's
//      segment cursors) and each key of the cut bin to the leader's tie buffer;
//   4. the leader takes the cut bin's best and ranks every segment.
// After the call only the leader may go on; no CTA touches another's shared
// memory after its last cluster barrier.
#pragma once
#include <cooperative_groups.h>

#include "st_internal.cuh"

namespace st {

struct ClusterCut {
    TopkCut t;
    uint32_t tpos;      // cut-bin keys sent to the leader
    int32_t lo, hi;     // this CTA's score range (step 0)
};

// keep(key) -> false drops a key (a post-filter); it must give the same answer
// in both passes. tmp: k keys, tie: tie_cap keys, out: next_pow2(k) keys, all
// in shared memory at the same offset in every CTA of the cluster. `compact`
// is called by the leader (all its threads) when the cut bin held more than
// tie_cap keys and filtering is on: it must move the cut bin's kept keys to
// the front of `keys` and return their count. Returns the number of sorted
// keys in the leader's out[] (min(kept, k)), -1 in the other CTAs.
template <int CS, int BLOCK, class Keep, class Compact>
__device__ int cluster_topk(cooperative_groups::cluster_group& cluster, const uint64_t* keys, int64_t n, int k,
                            bool range_known, int32_t lo, int32_t hi, bool filt, Keep keep, Compact compact,
                            uint64_t* tmp, uint64_t* tie, int tie_cap, uint64_t* out, SelectSmem& ss,
                            ClusterCut& cc, uint32_t* err)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int rank = int(cluster.block_rank());
    const int64_t s0 = n * rank / CS, s1 = n * (rank + 1) / CS;
    constexpr int U = 8;
    auto for_share = [&](auto&& fn) {
        for (int64_t base = s0; base < s1; base += int64_t(BLOCK) * U) {
            uint64_t v[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t i = base + int64_t(u) * BLOCK + tid;
                v[u] = i < s1 ? keys[i] : 0ull;
            }
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (base + int64_t(u) * BLOCK + tid < s1) fn(v[u]);
        }
    };
    if (!range_known) {
        // 0. the range of the kept keys' scores
        int32_t l = INT32_MAX, h = INT32_MIN;
        for_share([&](uint64_t key) {
            if (filt && !keep(key)) return;
            const int32_t sc = key_score(key);
            l = sc < l ? sc : l;
            h = sc > h ? sc : h;
        });
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            l = min(l, __shfl_xor_sync(0xffffffffu, l, off));
            h = max(h, __shfl_xor_sync(0xffffffffu, h, off));
        }
        if (lane == 0) {
            ss.red_lo[warp] = (unsigned long long)(uint32_t(l));
            ss.red_hi[warp] = (unsigned long long)(uint32_t(h));
        }
        __syncthreads();
        if (tid == 0) {
            l = INT32_MAX;
            h = INT32_MIN;
            for (int w = 0; w < BLOCK / 32; ++w) {
                l = min(l, int32_t(uint32_t(ss.red_lo[w])));
                h = max(h, int32_t(uint32_t(ss.red_hi[w])));
            }
            cc.lo = l;
            cc.hi = h;
        }
        cluster.sync();
        lo = INT32_MAX;
        hi = INT32_MIN;
#pragma unroll 1
        for (int r = 0; r < CS; ++r) {
            const ClusterCut* rc = cluster.map_shared_rank(&cc, r);
            lo = min(lo, rc->lo);
            hi = max(hi, rc->hi);
        }
        if (lo > hi) lo = hi = 0;  // no kept key at all
    }
    const uint32_t sh = topk_shift(lo, hi);
    // 1. this CTA's histogram
    for (int i = tid; i < kSelBins; i += BLOCK) ss.hist[i] = 0;
    if (rank == 0 && tid == 0) cc.tpos = 0;
    __syncthreads();
    for_share([&](uint64_t key) {
        if (!filt || keep(key)) atomicAdd(&ss.hist[topk_bin(key, lo, sh)], 1u);
    });
    cluster.sync();  // every CTA's histogram is complete (and every range read)
    // 2. the leader sums them and finds the cut
    if (rank == 0) {
        uint32_t local = 0;
        for (int i = tid; i < kSelBins; i += BLOCK) {
            uint32_t tot = ss.hist[i];
#pragma unroll 1
            for (int r = 1; r < CS; ++r) tot += cluster.map_shared_rank(&ss.hist[0], r)[i];
            ss.hist[i] = tot;
            local += tot;
        }
        uint32_t nk;
        block_excl_scan<BLOCK>(local, ss.part, nk);
        const TopkCut t = topk_cut_from_hist<BLOCK>(int64_t(nk), k, lo, sh, ss);
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
        for_share([&](uint64_t key) {
            const int b = topk_bin(key, lo, sh);
            if (b < cut) return;
            if (filt && !keep(key)) return;
            if (b > cut) {
                ltmp[atomicAdd(&cursor[b], 1u)] = key;
            } else {
                const uint32_t tp = atomicAdd(tpos, 1u);
                if (tp < uint32_t(tie_cap)) ltie[tp] = key;
            }
        });
    }
    cluster.sync();  // every key is in the leader's memory
    if (rank != 0) return -1;
    // 4. the leader: the cut bin's best, then every segment's order
    TopkCut t = cc.t;
    const uint64_t* tsrc = tie;
    if (t.tcount > tie_cap) {
        tsrc = nullptr;  // select over every key of the cut bin in global memory
        if (filt && t.m > t.above) {
            t.tcount = compact();
            tsrc = keys;
        }
    }
    topk_take_ties<BLOCK>(t, tsrc, keys, n, tmp, ss, err);
    topk_rank<BLOCK>(t, tmp, out, ss);
    return t.m;
}

// Launch a kernel with `cs` CTAs per cluster as a programmatic dependent launch.
template <typename... KArgs, typename... Args>
cudaError_t launch_dep_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, int cs, cudaStream_t s,
                               Args&&... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = unsigned(cs);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// CTAs per query cluster: enough to cover the SMs about twice at small
// batches, one CTA per query at large ones.
__host__ __forceinline__ int cluster_size_for(int B, int num_sms)
{
    if (B * 8 <= 2 * num_sms) return 8;
    if (B * 4 <= 2 * num_sms) return 4;
    if (B * 2 <= 2 * num_sms) return 2;
    return 1;
}

}  // namespace st
