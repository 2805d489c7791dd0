// Device helpers shared by the final top-k kernels (select.cu,
// select_cluster.cu): the exact overflow path, the query's score range, and
// the post-filter bookkeeping.
#pragma once
#include "st_internal.cuh"

namespace st {

// Exact overflow path: when the scan reserved more candidates for a query than
// its buffer holds, one CTA rescans that query's probed lists itself with the
// bounded buffer: whenever the buffer fills it keeps only the k best keys and
// from then on drops any key below the k-th, which can no longer enter the
// top-k. Exact for any input, with memory bounded by the capacity; slow, and
// used only on overflow. Returns the number of keys kept at the front of the
// query's candidate buffer.
template <int BLOCK>
__device__ int64_t overflow_path(const SearchArgs& a, int q, uint64_t* sortbuf, int pwk, int4* s_qv,
                                 SelectSmem& ss)
{
    __shared__ int32_t s_count;
    __shared__ uint64_t s_thr;
    const int d = a.d, np = d >> 4, W = a.W, k = a.k;
    uint64_t* buf = a.cand + int64_t(q) * a.cap;
    const int64_t cap = a.cap;  // host guarantees cap >= k + BLOCK
    for (int p = threadIdx.x; p < np; p += BLOCK)
        s_qv[p] = reinterpret_cast<const int4*>(a.queries + int64_t(q) * d)[p];
    const uint64_t m0 = a.qmasks[int64_t(q) * W];
    const uint64_t m1 = W > 1 ? a.qmasks[int64_t(q) * W + 1] : 0ull;
    if (threadIdx.x == 0) {
        s_count = 0;
        s_thr = 0;
    }
    __syncthreads();
    for (int p = 0; p < a.P; ++p) {
        const int L = a.probe[int64_t(q) * a.P + p];
        if (L < 0 || L >= a.nlist) {
            if (threadIdx.x == 0) set_error(a.err, kErrOverflowPath);
            continue;
        }
        // the list's chunks: its creation rows, then its append chunks
        const int t0 = a.chunk_start[L], t1 = a.chunk_start[L + 1];
        for (int t = t0; t < t1; ++t) {
            const int4 c = a.chunk_desc[t];  // {first row, plane block, rows, list}
            if (c.w != L || c.z < 0 || c.z > kWarpItems || c.x < 0 || int64_t(c.x) + c.z > a.n_rows) {
                if (threadIdx.x == 0) set_error(a.err, kErrOverflowPath);
                continue;
            }
            const int64_t o0 = c.x, o1 = int64_t(c.x) + c.z;
            for (int64_t base = o0; base < o1; base += BLOCK) {
                if (int64_t(s_count) + BLOCK > cap) {
                    // keep the k best, drop everything below them from now on
                    const int64_t cnt = s_count;
                    const uint64_t thr = block_select_threshold<BLOCK>(buf, cnt, k, ss, a.err);
                    const int32_t got = block_collect_ge<BLOCK>(buf, cnt, thr, sortbuf, pwk, ss);  // unsorted is fine here
                    if (threadIdx.x == 0 && got != k) set_error(a.err, kErrOverflowPath);
                    for (int i = threadIdx.x; i < k; i += BLOCK) buf[i] = sortbuf[i];
                    if (threadIdx.x == 0) {
                        s_count = k;
                        s_thr = thr;
                    }
                    __syncthreads();
                }
                const int64_t i = base + threadIdx.x;
                const uint64_t thr = s_thr;
                bool keep = false;
                uint64_t key = 0;
                if (i < o1) {
                    const uint64_t* sg = a.sigs + i * W;
                    bool pass = (sg[0] & m0) == m0;
                    if (W > 1) pass = pass && ((sg[1] & m1) == m1);
                    for (int alt = 0; alt < a.n_or && !pass; ++alt) {  // alternative masks: any one passes
                        const uint64_t* x = a.or_masks + (int64_t(q) * a.n_or + alt) * W;
                        pass = (sg[0] & x[0]) == x[0] && (W < 2 || (sg[1] & x[1]) == x[1]);
                    }
                    pass = pass && keep_item(a, q, i);
                    if (pass) {
                        const int4* rp = reinterpret_cast<const int4*>(a.items + i * d);
                        int32_t acc = 0;
                        for (int j = 0; j < np; ++j) acc = dot16(__ldg(rp + j), s_qv[j], acc);
                        key = pack_key(acc, uint32_t(i));
                        keep = key >= thr;
                    }
                }
                const unsigned bal = __ballot_sync(0xffffffffu, keep);
                if (bal) {
                    int32_t b0 = 0;
                    if ((threadIdx.x & 31) == 0) b0 = atomicAdd(&s_count, __popc(bal));
                    b0 = __shfl_sync(0xffffffffu, b0, 0);
                    if (keep) buf[b0 + __popc(bal & lanemask_lt())] = key;
                }
                __syncthreads();
            }
        }
    }
    return s_count;
}

// A range containing every score of query q: [-S, S], S = 128 sum_j |q_j|
// (the probe records -S); sh fits it into kSelBins bins.
__device__ __forceinline__ void query_range(const SearchArgs& a, int q, int32_t& lo, uint32_t& sh)
{
    lo = a.qscale[q].x;
    sh = topk_shift(lo, -lo);
}

// Candidates the chunked kernels handle for query q: all of them, unless the
// scan overflowed the query's buffer (the final kernel rescans those).
__device__ __forceinline__ int64_t chunked_count(const SearchArgs& a, int q)
{
    const int64_t n = a.cand_cnt[int64_t(q) * kCntStride];
    return n <= a.cap ? n : 0;
}

// Per-query words of score_rng used by the final top-k, after the scan's range:
// [2] cut-bin keys gathered, [3] chunks histogrammed, [4] cut bin, [5] keys
// above it, [6] keys in it, [7] longest output segment.
constexpr int kRngTie = 2, kRngDone = 3, kRngCut = 4, kRngAbove = 5, kRngTcount = 6, kRngMaxseg = 7;
constexpr int kRngKept = 9;  // candidates left after the post-filter

// The query's candidates that pass the post-filter (all of them without one).
__device__ __forceinline__ int64_t kept_count(const SearchArgs& a, int q)
{
    return (a.dead || a.qexclude) ? int64_t(__ldcg(a.score_rng + int64_t(q) * kCntStride + kRngKept))
                                  : chunked_count(a, q);
}

// Compact query q's candidates of the cut bin that pass the post-filter to
// the front of its candidate buffer (no longer read by anyone else) and
// return their count: one CTA, every thread's writes land only on positions
// already read.
template <int BLOCK>
__device__ int compact_cut_bin(const SearchArgs& a, int q, int64_t n, const TopkCut& t)
{
    __shared__ int c_cnt;
    uint64_t* keys = a.cand + int64_t(q) * a.cap;
    if (threadIdx.x == 0) c_cnt = 0;
    __syncthreads();
    for (int64_t base = 0; base < n; base += BLOCK) {
        const int64_t i = base + threadIdx.x;
        uint64_t key = 0;
        bool take = false;
        if (i < n) {
            key = keys[i];
            take = topk_bin(key, t.lo, t.sh) == t.cut && keep_item(a, q, key_id(key));
        }
        __syncthreads();  // this round's reads are done before any write
        if (take) keys[atomicAdd(&c_cnt, 1)] = key;
        __syncthreads();
    }
    return c_cnt;
}

}  // namespace st
