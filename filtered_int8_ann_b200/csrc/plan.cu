// Plan: invert the probe result (query -> lists) into list -> queries, so the
// scan reads each probed list once per batch however many queries probe it,
// and cut every distinct probed list into fixed-size work units
// (chunk of kWarpItems items) x (group of up to kQMax queries).
//
// One CTA. Steps: count the queries of every list; one block-wide exclusive
// scan gives each list its slice of the grouped query array and its first work
// unit; a second pass scatters the query ids into their list's slice. It also
// clears the per-query counters that the scan accumulates into and resets the
// scan's work counter, so a search needs no separate memset.
#include "st_internal.cuh"

namespace st {

template <int BLOCK>
__device__ void block_exclusive_scan3(int32_t v[3], int32_t out[3], int32_t total[3])
{
    __shared__ int32_t warp_tot[BLOCK / 32][3];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int32_t incl[3] = {v[0], v[1], v[2]};
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
#pragma unroll
        for (int c = 0; c < 3; ++c) {
            const int32_t t = __shfl_up_sync(0xffffffffu, incl[c], off);
            if (lane >= off) incl[c] += t;
        }
    }
    if (lane == 31)
        for (int c = 0; c < 3; ++c) warp_tot[warp][c] = incl[c];
    __syncthreads();
    if (warp == 0) {
        constexpr int NW = BLOCK / 32;
        int32_t w[3];
        for (int c = 0; c < 3; ++c) w[c] = lane < NW ? warp_tot[lane][c] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
#pragma unroll
            for (int c = 0; c < 3; ++c) {
                const int32_t t = __shfl_up_sync(0xffffffffu, w[c], off);
                if (lane >= off) w[c] += t;
            }
        }
        if (lane < NW)
            for (int c = 0; c < 3; ++c) warp_tot[lane][c] = w[c];  // inclusive per warp
    }
    __syncthreads();
    for (int c = 0; c < 3; ++c) {
        const int32_t before = warp > 0 ? warp_tot[warp - 1][c] : 0;
        out[c] = before + incl[c] - v[c];
        total[c] = warp_tot[BLOCK / 32 - 1][c];
    }
    __syncthreads();
}

template <int BLOCK>
__global__ void __launch_bounds__(BLOCK)
plan_kernel(SearchArgs a)
{
    const int nlist = a.nlist;
    const int npairs = a.B * a.P;
    const int tid = threadIdx.x;

    for (int L = tid; L < nlist; L += BLOCK) {
        a.list_cnt[L] = 0;
        a.list_fill[L] = 0;
    }
    for (int b = tid; b < a.B; b += BLOCK) {
        a.cand_cnt[b] = 0;
        a.eligible_cnt[b] = 0;
    }
    __syncthreads();
    for (int i = tid; i < npairs; i += BLOCK) {
        const int L = a.probe[i];
        if (L >= 0 && L < nlist) atomicAdd(&a.list_cnt[L], 1);
        else set_error(a.err, kErrSelectCount);
    }
    __syncthreads();

    // each thread owns a contiguous range of lists
    const int seg = (nlist + BLOCK - 1) / BLOCK;
    const int lo = min(nlist, tid * seg), hi = min(nlist, lo + seg);
    int32_t v[3] = {0, 0, 0};  // distinct lists with items, query slots, work units
    for (int L = lo; L < hi; ++L) {
        const int32_t c = a.list_cnt[L];
        const int64_t nL = a.offsets[L + 1] - a.offsets[L];
        v[1] += c;
        if (c > 0 && nL > 0) {
            v[0] += 1;
            v[2] += int32_t((nL + kWarpItems - 1) / kWarpItems) * ((c + kQMax - 1) / kQMax);
        }
    }
    int32_t ex[3], tot[3];
    block_exclusive_scan3<BLOCK>(v, ex, tot);
    for (int L = lo; L < hi; ++L) {
        const int32_t c = a.list_cnt[L];
        const int64_t nL = a.offsets[L + 1] - a.offsets[L];
        a.list_qstart[L] = ex[1];
        if (c > 0 && nL > 0) {
            const int j = ex[0];
            a.dl_list[j] = L;
            a.dl_qstart[j] = ex[1];
            a.dl_qcnt[j] = c;
            a.dl_ustart[j] = ex[2];
            ex[0] += 1;
            ex[2] += int32_t((nL + kWarpItems - 1) / kWarpItems) * ((c + kQMax - 1) / kQMax);
        }
        ex[1] += c;
    }
    if (tid == 0) {
        a.ctl->n_lists = tot[0];
        a.ctl->n_units = min(tot[2], a.max_units);
        if (tot[2] > a.max_units) set_error(a.err, kErrUnitTable);
        a.ctl->next_unit = 0;
        a.dl_ustart[tot[0]] = tot[2];
    }
    __syncthreads();
    for (int i = tid; i < npairs; i += BLOCK) {
        const int L = a.probe[i];
        if (L < 0 || L >= nlist) continue;
        const int pos = a.list_qstart[L] + atomicAdd(&a.list_fill[L], 1);
        a.qlist[pos] = i / a.P;
    }
}

// Expand: one self-contained 16-byte entry per work unit, so a scan warp needs
// a single load to know its rows and queries. Unit u of distinct list j covers
// chunk c = local % nchunks of the list and query group g = local / nchunks,
// where local = u - first unit of j (consecutive units walk down one list).
__global__ void __launch_bounds__(kExpandBlock)
expand_kernel(SearchArgs a)
{
    const int n_units = a.ctl->n_units;
    const int n_lists = a.ctl->n_lists;
    for (int u = blockIdx.x * kExpandBlock + threadIdx.x; u < n_units; u += gridDim.x * kExpandBlock) {
        int lo = 0, hi = n_lists - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (__ldg(a.dl_ustart + mid) <= u) lo = mid; else hi = mid - 1;
        }
        const int L = a.dl_list[lo];
        const int64_t o0 = a.offsets[L], o1 = a.offsets[L + 1];
        const int nchunks = int((o1 - o0 + kWarpItems - 1) / kWarpItems);
        const int local = u - a.dl_ustart[lo];
        const int g = local / nchunks, c = local - g * nchunks;
        const int qn = min(kQMax, a.dl_qcnt[lo] - g * kQMax);
        const int64_t ib = o0 + int64_t(c) * kWarpItems;
        const int len = int(min(o1 - ib, int64_t(kWarpItems)));
        if (local < 0 || qn <= 0 || len <= 0) {
            set_error(a.err, kErrUnitDecode);
            a.units[u] = make_int4(0, 0, 0, 0);
            continue;
        }
        a.units[u] = make_int4(int(ib), len, a.dl_qstart[lo] + g * kQMax, qn);
    }
}

cudaError_t launch_plan(const SearchArgs& a, int num_sms, cudaStream_t s)
{
    plan_kernel<kPlanBlock><<<1, kPlanBlock, 0, s>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    expand_kernel<<<num_sms * 2, kExpandBlock, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace st
