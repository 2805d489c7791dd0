// Final top-k: one CTA per query picks the k best candidate keys and writes
// them ordered by score descending, then item id ascending, padded with
// (id -1, score INT32_MIN) when fewer than k items were eligible.
//
// "Top-2048 with 64 probes and no recall loss" / a large candidate pool --
// SilverTorch: Index as Model, section on redesigning each stage as a pure
// PyTorch module, fused Int8 ANN paragraph; maximum top-k row of the cost
// efficiency table in the Spanish translation.
//
// The candidate keys of a query (written by the scan) are copied into shared
// memory when they fit; a radix select over the bits where they differ finds a
// threshold with exactly k keys at or above it; those keys are gathered and a
// bitonic network sorts them.
//
// Exact overflow path: when the scan reserved more candidates for a query than
// its buffer holds, this CTA rescans that query's probed lists itself with the
// bounded buffer: whenever the buffer fills it keeps only the k best keys and
// from then on drops any key below the k-th, which can no longer enter the
// top-k. Exact for any input, with memory bounded by the capacity; slow, and
// used only on overflow.
#include "st_internal.cuh"

namespace st {

template <int BLOCK>
__device__ int32_t select_into(const uint64_t* keys, int64_t n, int k, uint64_t* sortbuf, int pwk,
                               SelectSmem& ss, uint32_t* err, uint64_t* tmp)
{
    int32_t got;
    if (n > k) {
        const uint64_t thr = block_select_threshold<BLOCK>(keys, n, k, ss, err);
        got = block_collect_ge<BLOCK>(keys, n, thr, sortbuf, pwk, ss);
        if (threadIdx.x == 0 && got != k) set_error(err, kErrSelectCount);
    } else {
        got = block_collect_ge<BLOCK>(keys, n, 1ull, sortbuf, pwk, ss);
    }
    if (got > pwk) got = pwk;
    for (int i = got + threadIdx.x; i < pwk; i += BLOCK) sortbuf[i] = 0;
    __syncthreads();
    block_sort_desc_counting<BLOCK>(sortbuf, got, tmp, ss);
    return got;
}

// Histogram-guided threshold: the bin holding the k-th best score is found from
// the per-query histogram the scan built; every key of that bin or above is
// collected (about k plus one bin), and the exact threshold is selected among
// them only. Returns false (and leaves nothing) when the histogram does not
// match the keys or the collected set does not fit, so the caller falls back.
template <int BLOCK>
__device__ bool hist_guided_select(const SearchArgs& a, int q, const uint64_t* keys, int64_t n, int k,
                                   uint64_t* sortbuf, int pwk, uint64_t* buf, int buf_cap, SelectSmem& ss)
{
    __shared__ uint32_t s_cut_bin, s_cut_above;
    const uint32_t* h = a.hist + int64_t(q) * kHistBins;
    constexpr int PER = kHistBins / BLOCK > 0 ? kHistBins / BLOCK : 1;
    uint32_t c[PER];
    uint32_t local = 0;
    // thread t owns bins counted down from the top: kHistBins-1-(t*PER+j)
    for (int j = 0; j < PER; ++j) {
        const int bin = kHistBins - 1 - (int(threadIdx.x) * PER + j);
        c[j] = bin >= 0 ? h[bin] : 0u;
        local += c[j];
    }
    if (threadIdx.x == 0) {
        s_cut_bin = 0;
        s_cut_above = 0xFFFFFFFFu;
    }
    uint32_t total;
    const uint32_t excl = block_excl_scan<BLOCK>(local, ss.part, total);
    if (excl < uint32_t(k) && uint32_t(k) <= excl + local) {
        uint32_t acc = excl;
        for (int j = 0; j < PER; ++j) {
            if (acc + c[j] >= uint32_t(k)) {
                s_cut_bin = uint32_t(kHistBins - 1 - (int(threadIdx.x) * PER + j));
                s_cut_above = acc;
                break;
            }
            acc += c[j];
        }
    }
    __syncthreads();
    if (int64_t(total) != n || s_cut_above == 0xFFFFFFFFu) return false;
    // lowest score of the cut bin -> key threshold (every key of a score >= it)
    const int32_t s_lo = s_cut_bin == 0 ? INT32_MIN + 1 : int32_t((int64_t(s_cut_bin) << a.hshift) - a.smax);
    const uint64_t thr = pack_key(s_lo, 0xFFFFFFFFu);
    const int32_t got = block_collect_ge_wide<BLOCK>(keys, n, thr, buf, buf_cap, ss);
    if (got > buf_cap || got < k) return false;
    const uint64_t t2 = block_select_threshold<BLOCK>(buf, got, k, ss, a.err);
    const int32_t fin = block_collect_ge<BLOCK>(buf, got, t2, sortbuf, pwk, ss);
    if (threadIdx.x == 0 && fin != k) set_error(a.err, kErrSelectCount);
    for (int i = (fin < pwk ? fin : pwk) + threadIdx.x; i < pwk; i += BLOCK) sortbuf[i] = 0;
    __syncthreads();
    block_sort_desc_counting<BLOCK>(sortbuf, fin < pwk ? fin : pwk, buf, ss);  // buf's keys are no longer needed
    return true;
}

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
        const int64_t o0 = a.offsets[L], o1 = a.offsets[L + 1];
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
                if (pass) {
                    const int4* rp = reinterpret_cast<const int4*>(a.items + i * d);
                    int32_t acc = 0;
                    for (int t = 0; t < np; ++t) acc = dot16(__ldg(rp + t), s_qv[t], acc);
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
    return s_count;
}

template <int BLOCK>
__global__ void __launch_bounds__(BLOCK)
select_kernel(SearchArgs a)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ SelectSmem ss;
    const int q = blockIdx.x;
    const int k = a.k;
    const int pwk = next_pow2(k);
    uint64_t* sortbuf = reinterpret_cast<uint64_t*>(smem_raw);    // max(pwk, BLOCK) keys
    uint64_t* local = sortbuf + (pwk > BLOCK ? pwk : BLOCK);       // 16-byte aligned

    const uint32_t cnt = a.cand_cnt[int64_t(q) * kCntStride];
    const uint64_t* keys = a.cand + int64_t(q) * a.cap;
    int64_t n = cnt;
    const bool overflow = n > a.cap;
    if (overflow) n = overflow_path<BLOCK>(a, q, sortbuf, pwk, reinterpret_cast<int4*>(local), ss);
    bool done = false;
    if (!overflow && n > k) {
        // common case: the scan's histogram gives the cut; one pass over the
        // candidates in global memory collects about k keys into shared memory
        done = hist_guided_select<BLOCK>(a, q, keys, n, k, sortbuf, pwk, local, kSelectSmemKeys, ss);
    }
    if (!done && n <= kSelectSmemKeys) {
        // all of this thread's 16-byte copies in flight at once (cp.async)
        const int64_t n2 = (n + 1) >> 1;
        const ulonglong2* src2 = reinterpret_cast<const ulonglong2*>(keys);
        ulonglong2* dst2 = reinterpret_cast<ulonglong2*>(local);
        for (int64_t i = threadIdx.x; i < n2; i += BLOCK) cp_async16(dst2 + i, src2 + i);
        cp_async_commit();
        cp_async_wait_all();
        __syncthreads();
        if ((n & 1) && threadIdx.x == 0) local[n] = 0;  // the pair's second key was past the end
        __syncthreads();
        keys = local;
    }
    // the candidate area is free once the final keys are in sortbuf
    if (!done) select_into<BLOCK>(keys, n, k, sortbuf, pwk, ss, a.err, local);
    for (int r = threadIdx.x; r < k; r += BLOCK) {
        const uint64_t key = sortbuf[r];
        a.out_ids[int64_t(q) * k + r] = key_id(key);
        a.out_scores[int64_t(q) * k + r] = key_score(key);
    }
    if (threadIdx.x == 0 && a.out_eligible) a.out_eligible[q] = int64_t(a.eligible_cnt[int64_t(q) * (kCntStride / 2)]);
}

cudaError_t launch_select(const SearchArgs& a, cudaStream_t s)
{
    const int pwk = next_pow2(a.k);
    const size_t smem = size_t(pwk > kSelectBlock ? pwk : kSelectBlock) * 8 + size_t(kSelectSmemKeys) * 8;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(select_kernel<kSelectBlock>), 8,
                                     int(size_t(ST_MAX_K) * 8 + size_t(kSelectSmemKeys) * 8));
    if (e != cudaSuccess) return e;
    select_kernel<kSelectBlock><<<a.B, kSelectBlock, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace st
