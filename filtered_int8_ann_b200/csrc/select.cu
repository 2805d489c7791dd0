// Final top-k in global memory, for k above ST_SMALL_K and for batches of at
// most kChunkedMaxB queries (otherwise select_cluster.cu):
// the k best candidate keys of each query, ordered by score descending, then
// item id ascending, padded with (id -1, score INT32_MIN) when fewer than k
// items were eligible.
//
// A large result drawn from a large candidate pool -- SilverTorch: Index as
// Model, section on redesigning each stage as a pure PyTorch module, fused
// Int8 ANN paragraph; maximum top-k row of the cost efficiency table in the
// Spanish translation (a count in the hundreds of thousands).
//
// The candidates of every query are cut into chunks of kChunk keys, so that a
// query with millions of candidates is spread over every SM:
//   * select_hist_kernel: each chunk's keys go into a 2048-bin histogram of
//     their scores over the query's score range (recorded by the scan),
//     added into the query's histogram; the query's last chunk finds the cut
//     bin (the one holding the k-th best score) and each higher bin's output
//     segment;
//   * select_scatter_kernel: every chunk writes its keys of the bins above the
//     cut into their segments; the cut bin's keys are gathered aside;
//   * k <= ST_SMALL_K: select_kernel, one CTA per query, takes the cut bin's
//     best, orders every segment in shared memory and writes ids and scores
//     (or takes the exact overflow path when the scan's buffer overflowed);
//   * larger k: select_ties_kernel (one CTA per query) takes the cut bin's
//     best and select_rank_kernel (one thread per output position) ranks each
//     key in its segment and writes the id and score. The scan reserves room
//     for every row of the probed lists when k is this large, so there is no
//     overflow path there.
#include "select_common.cuh"

namespace st {

constexpr int kChunk = 4096;      // candidates per histogram / scatter item
constexpr int kChunkBlock = 512;
constexpr int kChunkedMaxB = 8;   // batches up to this size take the chunked kernels for any k

// pre[q] = first item of query q (items: chunks of kChunk candidates), pre[B] = total
template <int BLOCK>
__device__ void chunk_prefix(const SearchArgs& a, int* pre, uint32_t* part)
{
    const int B = a.B;
    const int per = (B + BLOCK - 1) / BLOCK;
    const int q0 = threadIdx.x * per;
    uint32_t local = 0;
    for (int j = 0; j < per; ++j)
        if (q0 + j < B) local += uint32_t((chunked_count(a, q0 + j) + kChunk - 1) / kChunk);
    uint32_t total;
    uint32_t run = block_excl_scan<BLOCK>(local, part, total);
    for (int j = 0; j < per; ++j)
        if (q0 + j < B) {
            pre[q0 + j] = int(run);
            run += uint32_t((chunked_count(a, q0 + j) + kChunk - 1) / kChunk);
        }
    if (threadIdx.x == 0) pre[B] = int(total);
    __syncthreads();
}

__device__ __forceinline__ int item_query(const int* pre, int B, int item)
{
    int lo = 0, hi = B - 1;  // the last q with pre[q] <= item
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pre[mid] <= item) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

__global__ void __launch_bounds__(kChunkBlock)
select_hist_kernel(SearchArgs a)
{
    dep_enter();
    extern __shared__ int pre[];  // [B + 1]
    __shared__ SelectSmem ss;
    __shared__ int s_last;
    chunk_prefix<kChunkBlock>(a, pre, ss.part);
    const int total = pre[a.B];
    uint32_t* h = ss.hist2;  // this chunk's histogram
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
        const int q = item_query(pre, a.B, item);
        const int64_t c0 = int64_t(item - pre[q]) * kChunk;
        const int64_t n = chunked_count(a, q);
        const int cnt = int(n - c0 < kChunk ? n - c0 : kChunk);
        int32_t lo;
        uint32_t sh;
        query_range(a, q, lo, sh);
        for (int i = threadIdx.x; i < kSelBins; i += kChunkBlock) h[i] = 0;
        __syncthreads();
        const uint64_t* keys = a.cand + int64_t(q) * a.cap + c0;
        constexpr int U = kChunk / kChunkBlock;
        uint64_t v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = u * kChunkBlock + threadIdx.x;
            v[u] = i < cnt ? keys[i] : 0ull;
        }
        const bool filt = a.dead || a.qexclude;
        int kept = 0;
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (u * kChunkBlock + int(threadIdx.x) < cnt && (!filt || keep_item(a, q, key_id(v[u])))) {
                atomicAdd(&h[topk_bin(v[u], lo, sh)], 1u);
                ++kept;
            }
        if (filt) {
            kept = __reduce_add_sync(0xffffffffu, kept);
            if ((threadIdx.x & 31) == 0 && kept) atomicAdd(a.score_rng + int64_t(q) * kCntStride + kRngKept, uint32_t(kept));
        }
        __syncthreads();
        uint32_t* gh = a.sel_hist + int64_t(q) * kSelBins;
        for (int i = threadIdx.x; i < kSelBins; i += kChunkBlock)
            if (h[i]) atomicAdd(&gh[i], h[i]);
        // the query's last chunk to finish (one counter, no waiting) finds the
        // cut and writes each bin's segment start as the scatter's cursor
        __threadfence();
        __syncthreads();
        uint32_t* rng = a.score_rng + int64_t(q) * kCntStride;
        if (threadIdx.x == 0) s_last = atomicAdd(&rng[kRngDone], 1u) == uint32_t((n + kChunk - 1) / kChunk - 1);
        __syncthreads();
        if (s_last) {
            __threadfence();
            for (int i = threadIdx.x; i < kSelBins; i += kChunkBlock) ss.hist[i] = __ldcg(gh + i);
            __syncthreads();
            const TopkCut t = topk_cut_from_hist<kChunkBlock>(kept_count(a, q), a.k, lo, sh, ss);
            uint32_t* cur = a.sel_cursor + int64_t(q) * kSelBins;
            for (int i = threadIdx.x; i < kSelBins; i += kChunkBlock) cur[i] = ss.hist2[i];
            if (threadIdx.x == 0) {
                rng[kRngCut] = uint32_t(t.cut);
                rng[kRngAbove] = uint32_t(t.above);
                rng[kRngTcount] = uint32_t(t.tcount);
                rng[kRngMaxseg] = uint32_t(t.maxseg);
            }
        }
        __syncthreads();
    }
}

__global__ void __launch_bounds__(kChunkBlock)
select_scatter_kernel(SearchArgs a)
{
    dep_enter();
    extern __shared__ int pre[];  // [B + 1]
    __shared__ uint32_t part[32];
    chunk_prefix<kChunkBlock>(a, pre, part);
    const int total = pre[a.B];
    const int k = a.k;
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
        const int q = item_query(pre, a.B, item);
        const int64_t c0 = int64_t(item - pre[q]) * kChunk;
        const int64_t n = chunked_count(a, q);
        const int cnt = int(n - c0 < kChunk ? n - c0 : kChunk);
        int32_t lo;
        uint32_t sh;
        query_range(a, q, lo, sh);
        const int cut = int(a.score_rng[int64_t(q) * kCntStride + kRngCut]);
        const uint64_t* keys = a.cand + int64_t(q) * a.cap + c0;
        uint32_t* cur = a.sel_cursor + int64_t(q) * kSelBins;
        uint64_t* out = a.sel_out + int64_t(q) * k;
        uint64_t* tie = a.sel_tie + int64_t(q) * kSelTieCap;
        uint32_t* tcnt = a.score_rng + int64_t(q) * kCntStride + kRngTie;
        constexpr int U = kChunk / kChunkBlock;
        uint64_t v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = u * kChunkBlock + threadIdx.x;
            v[u] = i < cnt ? keys[i] : 0ull;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (u * kChunkBlock + int(threadIdx.x) >= cnt) continue;
            if ((a.dead || a.qexclude) && !keep_item(a, q, key_id(v[u]))) continue;
            const int b = topk_bin(v[u], lo, sh);
            if (b > cut) {
                out[atomicAdd(&cur[b], 1u)] = v[u];
            } else if (b == cut) {
                const uint32_t tp = atomicAdd(tcnt, 1u);
                if (tp < uint32_t(kSelTieCap)) tie[tp] = v[u];
            }
        }
        __syncthreads();
    }
}

// Finish of the chunked path for k <= ST_SMALL_K: one CTA per query takes
// the cut bin's best, orders every segment and writes ids and scores; a query
// whose candidates overflowed the scan's buffer takes the exact overflow path.
constexpr int kSelectTieCapSmem = 1024;

template <int BLOCK>
__global__ void __launch_bounds__(BLOCK)
select_kernel(SearchArgs a, int stage_cap)
{
    dep_enter();
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ SelectSmem ss;
    const int q = blockIdx.x;
    const int k = a.k;
    const int pwk = next_pow2(k);
    // shared layout: [tmp k keys, rounded up to even][tie kSelectTieCapSmem keys]
    // [stage_cap keys (>= next_pow2(k)): staged candidates / the output]
    uint64_t* tmp = reinterpret_cast<uint64_t*>(smem_raw);
    uint64_t* tie = tmp + ((k + 1) & ~1);
    uint64_t* stage = tie + kSelectTieCapSmem;

    const uint32_t cnt = a.cand_cnt[int64_t(q) * kCntStride];
    int64_t n = cnt;
    int m = 0;
    uint64_t* out = stage;
    if (n > a.cap) {
        // the scan overflowed this query's buffer: rescan exactly, then select
        // from the kept keys here
        n = overflow_path<BLOCK>(a, q, stage, pwk, reinterpret_cast<int4*>(tie), ss);
        const uint64_t* keys = a.cand + int64_t(q) * a.cap;
        if (n <= stage_cap) {
            for (int64_t i = threadIdx.x; i < n; i += BLOCK) stage[i] = keys[i];
            __syncthreads();
            keys = stage;
        } else {
            out = a.cand + int64_t(q) * a.cap;  // cap >= n > stage_cap >= next_pow2(k)
        }
        m = block_topk_sorted<BLOCK>(keys, n, k, out, tmp, tie, kSelectTieCapSmem, false, 0, 0, ss, a.err);
    } else if (n > 0) {
        // the chunked kernels grouped the keys above the cut bin by bin
        int32_t lo;
        uint32_t sh;
        query_range(a, q, lo, sh);
        // the histogram kernel's cut; after the scatter the cursor of bin b + 1
        // (the next higher bin) stands at the end of its segment, which is
        // where bin b's segment starts
        const uint32_t* rng = a.score_rng + int64_t(q) * kCntStride;
        TopkCut t;
        t.lo = lo;
        t.sh = sh;
        t.cut = int(rng[kRngCut]);
        t.above = int(rng[kRngAbove]);
        t.tcount = int(rng[kRngTcount]);
        t.maxseg = int(rng[kRngMaxseg]);
        const int64_t nk = kept_count(a, q);
        t.m = nk < k ? int(nk) : k;
        const uint32_t* cur = a.sel_cursor + int64_t(q) * kSelBins;
        for (int i = threadIdx.x; i < kSelBins; i += BLOCK) ss.hist2[i] = i + 1 < kSelBins ? cur[i + 1] : 0u;
        const uint64_t* gout = a.sel_out + int64_t(q) * k;
        for (int i = threadIdx.x; i < t.above; i += BLOCK) tmp[i] = gout[i];
        const uint64_t* gtie = a.sel_tie + int64_t(q) * kSelTieCap;
        const uint64_t* tsrc = nullptr;  // the cut bin's keys, if they were all kept
        if (t.tcount <= kSelectTieCapSmem) {
            for (int i = threadIdx.x; i < t.tcount; i += BLOCK) tie[i] = gtie[i];
            tsrc = tie;
        } else if (t.tcount <= kSelTieCap) {
            tsrc = gtie;
        }
        __syncthreads();
        if (tsrc == nullptr && (a.dead || a.qexclude) && t.m > t.above) {
            // the cut bin was too large to keep aside: its filtered keys, compacted
            const int nt = compact_cut_bin<BLOCK>(a, q, n, t);
            t.tcount = nt;
            tsrc = a.cand + int64_t(q) * a.cap;
        }
        topk_take_ties<BLOCK>(t, tsrc, a.cand + int64_t(q) * a.cap, n, tmp, ss, a.err);
        topk_rank<BLOCK>(t, tmp, out, ss);
        m = t.m;
    }
    for (int r = threadIdx.x; r < k; r += BLOCK) {
        const uint64_t key = r < m ? out[r] : 0ull;  // key 0 reads as (id -1, INT32_MIN)
        a.out_ids[int64_t(q) * k + r] = key == 0ull ? -1 : key_id(key) + a.id_offset;
        a.out_scores[int64_t(q) * k + r] = key_score(key);
    }
    if (threadIdx.x == 0 && a.out_eligible) a.out_eligible[q] = int64_t(a.eligible_cnt[int64_t(q) * (kCntStride / 2)]);
    if (threadIdx.x == 0 && a.out_cands) a.out_cands[q] = int64_t(cnt);
}

// ----------------------------------------------------------------------------
// k above ST_SMALL_K: the same histogram and scatter, then the cut bin's best
// per query and every key's rank in its segment, all in global memory.
// ----------------------------------------------------------------------------
template <int BLOCK>
__global__ void __launch_bounds__(BLOCK)
select_ties_kernel(SearchArgs a)
{
    dep_enter();
    __shared__ SelectSmem ss;
    const int q = blockIdx.x;
    const int k = a.k;
    const int64_t n = a.cand_cnt[int64_t(q) * kCntStride];
    if (n <= 0) return;
    int32_t lo;
    uint32_t sh;
    query_range(a, q, lo, sh);
    const uint32_t* rng = a.score_rng + int64_t(q) * kCntStride;
    TopkCut t;
    t.lo = lo;
    t.sh = sh;
    t.cut = int(rng[kRngCut]);
    t.above = int(rng[kRngAbove]);
    t.tcount = int(rng[kRngTcount]);
    t.maxseg = int(rng[kRngMaxseg]);
    const int64_t nk = kept_count(a, q);
    t.m = nk < k ? int(nk) : k;
    const uint64_t* gtie = t.tcount <= kSelTieCap ? a.sel_tie + int64_t(q) * kSelTieCap : nullptr;
    if (gtie == nullptr && (a.dead || a.qexclude) && t.m > t.above) {
        t.tcount = compact_cut_bin<BLOCK>(a, q, n, t);  // the cut bin's filtered keys
        gtie = a.cand + int64_t(q) * a.cap;
    }
    topk_take_ties<BLOCK>(t, gtie, a.cand + int64_t(q) * a.cap, n, a.sel_out + int64_t(q) * k, ss, a.err);
}

// One thread per output position: the key at position p of the query's
// bin-grouped keys goes to its segment start + its rank in the segment.
__global__ void __launch_bounds__(256)
select_rank_kernel(SearchArgs a)
{
    dep_enter();
    const int k = a.k;
    const int64_t idx = int64_t(blockIdx.x) * 256 + threadIdx.x;
    if (idx >= int64_t(a.B) * k) return;
    const int q = int(idx / k);
    const int p = int(idx - int64_t(q) * k);
    const int64_t n = a.cand_cnt[int64_t(q) * kCntStride] > 0 ? kept_count(a, q) : 0;
    const int m = n < k ? int(n) : k;
    if (p == 0 && a.out_eligible) a.out_eligible[q] = int64_t(a.eligible_cnt[int64_t(q) * (kCntStride / 2)]);
    if (p == 0 && a.out_cands) a.out_cands[q] = int64_t(a.cand_cnt[int64_t(q) * kCntStride]);
    if (p >= m) {
        a.out_ids[idx] = -1;
        a.out_scores[idx] = INT32_MIN;
        return;
    }
    const uint64_t* keys = a.sel_out + int64_t(q) * k;
    const uint64_t key = keys[p];
    const int above = int(a.score_rng[int64_t(q) * kCntStride + kRngAbove]);
    int beg, end;
    if (p >= above) {
        beg = above;
        end = m;
    } else {
        int32_t lo;
        uint32_t sh;
        query_range(a, q, lo, sh);
        const int b = topk_bin(key, lo, sh);
        const uint32_t* cur = a.sel_cursor + int64_t(q) * kSelBins;  // after the scatter: bin ends
        beg = b + 1 < kSelBins ? int(cur[b + 1]) : 0;
        end = int(cur[b]);
    }
    int r = 0;
    for (int j = beg; j < end; ++j) r += keys[j] > key ? 1 : 0;
    const int64_t o = int64_t(q) * k + beg + r;
    a.out_ids[o] = key_id(key) + a.id_offset;
    a.out_scores[o] = key_score(key);
}

size_t select_smem(int k, int* stage_cap)
{
    const size_t budget = 208 * 1024;
    const size_t fixed = (size_t((k + 1) & ~1) + kSelectTieCapSmem) * 8;
    *stage_cap = int((budget - fixed) / 8) & ~1;
    return budget;
}

cudaError_t launch_select_cluster(const SearchArgs& a, int num_sms, cudaStream_t s);

bool select_reads_bins(int B, int k) { return k <= ST_SMALL_K && B > kChunkedMaxB; }

cudaError_t launch_select(const SearchArgs& a, int num_sms, cudaStream_t s)
{
    // a batch of few queries may hold millions of candidates per query (a
    // flat scan): spread them over the whole GPU with the chunked kernels;
    // otherwise one cluster per query does it in one launch
    if (select_reads_bins(a.B, a.k)) return launch_select_cluster(a, num_sms, s);
    // the attribute is set once per device: give it the largest size any batch uses
    constexpr int kPreSmemMax = 160 * 1024;
    const size_t pre_bytes = size_t(a.B + 1) * 4;
    if (pre_bytes > size_t(kPreSmemMax)) return cudaErrorInvalidValue;
    const int grid = 3 * num_sms;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(select_hist_kernel), kPreSmemMax);
    if (e != cudaSuccess) return e;
    e = launch_dep(select_hist_kernel, dim3(grid), dim3(kChunkBlock), pre_bytes, s, a);
    if (e != cudaSuccess) return e;
    e = ensure_smem_attr(reinterpret_cast<const void*>(select_scatter_kernel), kPreSmemMax);
    if (e != cudaSuccess) return e;
    e = launch_dep(select_scatter_kernel, dim3(grid), dim3(kChunkBlock), pre_bytes, s, a);
    if (e != cudaSuccess) return e;
    if (a.k <= ST_SMALL_K) {
        int stage_cap = 0;
        const size_t smem = select_smem(a.k, &stage_cap);
        e = ensure_smem_attr(reinterpret_cast<const void*>(select_kernel<kSelectBlock>), int(smem));
        if (e != cudaSuccess) return e;
        return launch_dep(select_kernel<kSelectBlock>, dim3(a.B), dim3(kSelectBlock), smem, s, a, stage_cap);
    }
    e = launch_dep(select_ties_kernel<kSelectBlock>, dim3(a.B), dim3(kSelectBlock), 0, s, a);
    if (e != cudaSuccess) return e;
    const int64_t threads = int64_t(a.B) * a.k;
    return launch_dep(select_rank_kernel, dim3(unsigned((threads + 255) / 256)), dim3(256), 0, s, a);
}

}  // namespace st
