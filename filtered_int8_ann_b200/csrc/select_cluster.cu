// Final top-k for batches of more than 8 queries and k <= ST_SMALL_K: one
// thread-block cluster of CS CTAs per query -- the k best candidate keys of
// each query, score descending then item id ascending, padded with id -1 /
// INT32_MIN (SilverTorch: Index as Model, section on redesigning each stage
// as a pure PyTorch module, fused Int8 ANN paragraph: a large result pool;
// maximum top-k row of the compute cost efficiency table in the Spanish
// translation).
//
// The scans counted every candidate key they wrote in the query's score bins
// (kTcBins bins over its possible range [-S, S]), so the bin holding the k-th
// best score -- the cut -- is known before any key is read, and so is the
// number of keys at or above it (k plus at most the cut bin's keys):
//   1. every CTA reads the bins and finds the cut (no communication): a
//      suffix scan over the lanes' bin sums finds the lane holding it, a
//      second one over that lane's bins the bin itself;
//   2. each CTA reads its share of the keys once and sends the keys at or
//      above the cut straight into the leader's shared memory (distributed
//      shared memory; one atomic per warp for their positions);
//   3. the leader sorts those few keys in its own shared memory (a counting
//      sort over their own score range) and writes the k best.
// Two cluster barriers in all. When the keys above the cut would not fit the
// leader's buffer (many equal or close scores), the general cluster selection
// (cluster_topk.cuh) runs over the query's keys at or above the cut instead.
// With deletions or exclude masks the
// scans' counts include keys the post-filter drops, so those searches take
// the general cluster selection (cluster_topk.cuh) with the post-filter
// applied to every key; a query whose candidates overflowed the scan's buffer
// takes the exact overflow path in the leader alone. Both exits happen before
// any cluster barrier and are the same for every CTA of the cluster.
#include "cluster_topk.cuh"
#include "select_common.cuh"

namespace cg = cooperative_groups;

namespace st {

constexpr int kCBlock = 512;
constexpr int kCTieCap = 4096;   // cut-bin keys of the general (post-filter) path

// Keys at or above the cut the leader can hold.
__host__ __device__ __forceinline__ int cl_buf_cap(int k)
{
    const int c = 2 * next_pow2(k);
    return c < 1024 ? 1024 : c;
}

__host__ __device__ __forceinline__ size_t select_cluster_smem(int k)
{
    const size_t ke = size_t((k + 1) & ~1), pw = size_t(next_pow2(k));
    const size_t fast = 2 * size_t(cl_buf_cap(k));  // gathered keys, then the sort's scratch
    const size_t general = ke + kCTieCap + pw;
    return (fast > general ? fast : general) * 8;
}

// The rare paths, kept out of line so that they do not crowd the common one's
// registers: the exact overflow path (the leader alone) ...
__device__ __noinline__ int cl_overflow(const SearchArgs& a, int q, int k, uint64_t* keys, uint64_t* smem_keys,
                                        SelectSmem& ss)
{
    uint64_t* tmp = smem_keys;
    uint64_t* tie = tmp + ((k + 1) & ~1);
    uint64_t* out = tie + kCTieCap;
    const int64_t nk = overflow_path<kCBlock>(a, q, out, next_pow2(k), reinterpret_cast<int4*>(tie), ss);
    // the kept keys are at the front of the candidate buffer
    return block_topk_sorted<kCBlock>(keys, nk, k, out, tmp, tie, kCTieCap, false, 0, 0, ss, a.err);
}

// ... and the general cluster selection over the keys in [lo, S] (all of
// them through the post-filter when filt), for the post-filter and for many
// keys at or above the cut.
template <int CS>
__device__ __noinline__ int cl_general(const SearchArgs& a, int q, int k, int64_t n, uint64_t* keys, bool filt,
                                       int32_t lo, int32_t hi, uint64_t* smem_keys, SelectSmem& ss, ClusterCut& cc)
{
    cooperative_groups::cluster_group cluster = cooperative_groups::this_cluster();
    uint64_t* tmp = smem_keys;
    uint64_t* tie = tmp + ((k + 1) & ~1);
    uint64_t* out = tie + kCTieCap;
    auto keep = [&](uint64_t key) { return key_score(key) >= lo && (!filt || keep_item(a, q, key_id(key))); };
    auto compact = [&]() { return compact_cut_bin<kCBlock>(a, q, n, cc.t); };
    return cluster_topk<CS, kCBlock>(cluster, keys, n, k, true, lo, hi, true, keep, compact, tmp, tie, kCTieCap, out,
                                     ss, cc, a.err);
}

template <int CS>
__global__ void __launch_bounds__(kCBlock)
select_cluster_kernel(const __grid_constant__ SearchArgs a)
{
    dep_enter();
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = int(cluster.block_rank());
    const int q = int(blockIdx.x) / CS;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ SelectSmem ss;
    __shared__ ClusterCut cc;
    __shared__ int s_cut;
    __shared__ uint32_t s_m, s_cnt;
    const int k = a.k;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    const uint32_t cnt = a.cand_cnt[int64_t(q) * kCntStride];
    const int64_t n = cnt;
    uint64_t* keys = a.cand + int64_t(q) * a.cap;
    const bool filt = a.dead || a.qexclude;
    const int2 sc = a.qscale[q];  // {-S, shift of the scans' bins}
    int m = 0;
    uint64_t* out;

    if (n > a.cap || n == 0) {
        // the scan overflowed this query's buffer, or no candidate: the
        // leader alone, and no cluster barrier
        if (rank != 0) return;
        out = reinterpret_cast<uint64_t*>(smem_raw) + ((k + 1) & ~1) + kCTieCap;
        if (n > 0) m = cl_overflow(a, q, k, keys, reinterpret_cast<uint64_t*>(smem_raw), ss);
    } else if (filt) {
        // general path: every key through the post-filter
        out = reinterpret_cast<uint64_t*>(smem_raw) + ((k + 1) & ~1) + kCTieCap;
        m = cl_general<CS>(a, q, k, n, keys, true, sc.x, -sc.x, reinterpret_cast<uint64_t*>(smem_raw), ss, cc);
        if (m < 0) return;  // not the leader
    } else {
        const int cap = cl_buf_cap(k);
        uint64_t* buf = reinterpret_cast<uint64_t*>(smem_raw);   // [cap] keys at or above the cut (leader)
        out = buf + cap;                                         // [cap] the leader's sort scratch
        // the leader's counter starts at zero; the cluster barrier that makes
        // it (and every CTA's start) visible is awaited only before the
        // first remote access
        if (rank == 0 && tid == 0) s_cnt = 0;
        asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
        // 1. the cut: the highest bin with at least min(n, k) keys at or above it
        constexpr int kPer = kTcBins / 32;  // bins per lane
        if (warp == 0) {
            const uint4* h = reinterpret_cast<const uint4*>(a.qhist + int64_t(q) * kTcBins) + lane * (kPer / 4);
            uint32_t tot = 0;
#pragma unroll
            for (int i = 0; i < kPer / 4; ++i) {
                const uint4 x = __ldcg(h + i);
                tot += x.x + x.y + x.z + x.w;
            }
            uint32_t incl = tot;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const uint32_t o = __shfl_down_sync(0xffffffffu, incl, off);
                if (lane + off < 32) incl += o;
            }
            const uint32_t want = n < k ? uint32_t(n) : uint32_t(k);
            const uint32_t above = incl - tot;  // keys in the bins above this lane's
            const unsigned found = __ballot_sync(0xffffffffu, above < want && incl >= want);
            if (found == 0u) {  // cannot happen: the bins hold all n keys
                if (lane == 0) {
                    s_cut = 0;
                    s_m = 0xFFFFFFFFu;
                }
            } else {
                // the lane L holding the cut: the whole warp reads its kPer bins
                // (one per lane) and finds the highest bin with at least `want`
                // keys at or above it by a suffix scan
                static_assert(kPer == 32, "one bin per lane");
                const int L = __ffs(found) - 1;
                const uint32_t runL = __shfl_sync(0xffffffffu, above, L);
                const uint32_t v = __ldcg(a.qhist + int64_t(q) * kTcBins + kPer * L + lane);
                uint32_t suf = v;  // keys in bins lane .. kPer - 1 of lane L's
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const uint32_t o = __shfl_down_sync(0xffffffffu, suf, off);
                    if (lane + off < 32) suf += o;
                }
                const unsigned ok = __ballot_sync(0xffffffffu, runL + suf >= want);
                const int j = 31 - __clz(ok);  // ok != 0: lane 0 sees every key of lane L's bins
                const uint32_t at = __shfl_sync(0xffffffffu, runL + suf, j);
                if (lane == 0) {
                    s_cut = kPer * L + j;
                    s_m = at;
                }
            }
        }
        __syncthreads();
        const int cut = s_cut;
        const uint32_t mt = s_m;
        const int32_t T = sc.x + (cut << sc.y);  // lowest score of the cut bin
        asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
        if (mt > uint32_t(cap)) {
            // too many keys at or above the cut (many equal or close scores):
            // the general cluster selection over all of them
            out = reinterpret_cast<uint64_t*>(smem_raw) + ((k + 1) & ~1) + kCTieCap;
            m = cl_general<CS>(a, q, k, n, keys, false, T, -sc.x, reinterpret_cast<uint64_t*>(smem_raw), ss, cc);
            if (m < 0) return;  // not the leader
        } else {
            uint32_t* lcnt = cluster.map_shared_rank(&s_cnt, 0);
            uint64_t* lbuf = cluster.map_shared_rank(buf, 0);
            // 2. this CTA's share of the keys; those at or above the cut go to
            // the leader. Shares start on even keys and are read as 16-byte
            // pairs, eight pairs in flight per thread (the query's buffer is
            // 256-byte aligned); an odd last key is read on its own.
            const int64_t s0 = (n * rank / CS) & ~int64_t(1);
            const int64_t s1 = rank == CS - 1 ? n : ((n * (rank + 1) / CS) & ~int64_t(1));
            const ulonglong2* kp = reinterpret_cast<const ulonglong2*>(keys);
            auto push = [&](bool take, uint64_t key) {
                const unsigned bal = __ballot_sync(0xffffffffu, take);
                if (!bal) return;
                uint32_t p0 = 0;
                if (lane == 0) p0 = atomicAdd(lcnt, uint32_t(__popc(bal)));
                p0 = __shfl_sync(0xffffffffu, p0, 0);
                const uint32_t pos = p0 + __popc(bal & lanemask_lt());
                if (take && pos < uint32_t(cap)) lbuf[pos] = key;
            };
            constexpr int U = 8;
            const int64_t e0 = s0 >> 1, e1 = s1 >> 1;  // whole pairs of the share
            for (int64_t base = e0; base < e1; base += int64_t(kCBlock) * U) {
                ulonglong2 v[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int64_t e = base + int64_t(u) * kCBlock + tid;
                    v[u] = e < e1 ? kp[e] : make_ulonglong2(0ull, 0ull);
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const bool in = base + int64_t(u) * kCBlock + tid < e1;
                    push(in && key_score(v[u].x) >= T, v[u].x);
                    push(in && key_score(v[u].y) >= T, v[u].y);
                }
            }
            if (s1 & 1) {  // the odd last key (last CTA only)
                const uint64_t key = warp == 0 ? keys[s1 - 1] : 0ull;
                if (warp == 0) push(lane == 0 && key_score(key) >= T, key);
            }
            cluster.sync();  // every key at or above the cut is in the leader's memory
            if (rank != 0) return;
            // 3. the leader: the k best of them, sorted
            const uint32_t got = s_cnt;
            if (tid == 0 && got != mt) set_error(a.err, kErrSelectCount);
            const int nb = int(got < uint32_t(cap) ? got : uint32_t(cap));
            // every gathered key is at or above the cut, and there are few of
            // them: sort them all (counting sort over their own score range;
            // out[] and what follows it serve as its scratch) and keep the k best
            block_sort_desc_counting<kCBlock>(buf, nb, out, ss);
            m = nb < k ? nb : k;
            out = buf;
        }
    }
    for (int r = tid; r < k; r += kCBlock) {
        const uint64_t key = r < m ? out[r] : 0ull;  // key 0 reads as (id -1, INT32_MIN)
        a.out_ids[int64_t(q) * k + r] = key == 0ull ? -1 : key_id(key) + a.id_offset;
        a.out_scores[int64_t(q) * k + r] = key_score(key);
    }
    if (tid == 0 && a.out_eligible) a.out_eligible[q] = int64_t(a.eligible_cnt[int64_t(q) * (kCntStride / 2)]);
    if (tid == 0 && a.out_cands) a.out_cands[q] = int64_t(cnt);
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
