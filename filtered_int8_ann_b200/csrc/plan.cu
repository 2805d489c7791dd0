// Plan: invert the probe result (query -> lists) into list -> query slots, so
// the scan reads each probed list once per batch however many queries probe
// it, and cut every probed list into warp work units of kWarpItems rows x a
// group of up to kQMax queries. One 16-byte unit entry {first row, rows, first
// query slot, queries} is all a scan warp needs.
//
// Multi-CTA without any grid-wide wait: CTA c owns the list range
// [c*nlist/G, (c+1)*nlist/G). Every CTA first reduces the per-list counts over
// all lists (vectorised, from L2) to get the slot and unit offsets at the start
// of its range and the grand total; it then scans its own lists, writes their
// slot starts and unit entries, and scatters the (query, list) pairs whose
// list it owns into the slot arrays (query id and that query's mask words, so
// the scan reads a slot with one load instead of two dependent ones). The
// per-list query counts were accumulated by the probe kernel into a zeroed
// array.
#include "st_internal.cuh"

namespace st {

template <int BLOCK>
__device__ __forceinline__ void block_sum3(long long v[3], long long* red /*[3][BLOCK/32]*/)
{
    constexpr int NW = BLOCK / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int c = 0; c < 3; ++c) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v[c] += __shfl_xor_sync(0xffffffffu, v[c], off);
        if (lane == 0) red[c * NW + warp] = v[c];
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < 3; ++c) {
        long long t = 0;
        for (int w = 0; w < NW; ++w) t += red[c * NW + w];
        v[c] = t;
    }
    __syncthreads();
}

__device__ __forceinline__ long long units_of(int32_t cnt, int32_t nch)
{
    return cnt > 0 ? (long long)nch * ((cnt + kQMax - 1) / kQMax) : 0;
}

template <int BLOCK>
__global__ void __launch_bounds__(BLOCK)
plan_kernel(SearchArgs a)
{
    __shared__ long long s_red[3 * (BLOCK / 32)];
    __shared__ uint32_t s_part[32];
    __shared__ int32_t s_uex[BLOCK + 1];
    __shared__ int32_t s_qex[BLOCK];
    __shared__ int32_t s_cnt[BLOCK];
    __shared__ int32_t s_nch[BLOCK];
    __shared__ long long s_off0[BLOCK];
    __shared__ long long s_off1[BLOCK];

    const int tid = threadIdx.x;
    const int nlist = a.nlist;
    const int G = gridDim.x, c = blockIdx.x;
    const int L0 = int((long long)c * nlist / G), L1 = int((long long)(c + 1) * nlist / G);

    // pass A: slot / unit offsets before L0, and the unit total (list_cnt is
    // padded with zeros to a multiple of 4 entries)
    long long v[3] = {0, 0, 0};  // slots before L0, units before L0, units total
    const int n4 = (nlist + 3) >> 2;
    const int4* cnt4 = reinterpret_cast<const int4*>(a.list_cnt);
#pragma unroll 4
    for (int i = tid; i < n4; i += BLOCK) {
        const int4 q = cnt4[i];
        const int cs[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int L = 4 * i + j;
            if (cs[j] == 0 || L >= nlist) continue;
            const long long u = units_of(cs[j], a.nchunks[L]);
            if (L < L0) {
                v[0] += cs[j];
                v[1] += u;
            }
            v[2] += u;
        }
    }
    block_sum3<BLOCK>(v, s_red);
    const long long total_units = v[2];
    if (c == 0 && tid == 0) {
        a.ctl->n_units = int(total_units < a.max_units ? total_units : a.max_units);
        if (total_units > a.max_units) set_error(a.err, kErrUnitTable);
    }

    // pass B: scan the owned lists tile by tile, write slot starts and units
    long long qbase = v[0], ubase = v[1];
    for (int t0 = L0; t0 < L1; t0 += BLOCK) {
        const int L = t0 + tid;
        int32_t cnt = 0, nch = 0;
        long long o0 = 0, o1 = 0;
        if (L < L1) {
            cnt = a.list_cnt[L];
            if (cnt > 0) {
                nch = a.nchunks[L];
                o0 = a.offsets[L];
                o1 = a.offsets[L + 1];
            }
        }
        const uint32_t u = uint32_t(units_of(cnt, nch));
        uint32_t qtot, utot;
        const uint32_t qex = block_excl_scan<BLOCK>(uint32_t(cnt), s_part, qtot);
        const uint32_t uex = block_excl_scan<BLOCK>(u, s_part, utot);
        if (L < L1) a.list_qstart[L] = int32_t(qbase + qex);
        s_uex[tid] = int32_t(uex);
        s_qex[tid] = int32_t(qex);
        s_cnt[tid] = cnt;
        s_nch[tid] = nch;
        s_off0[tid] = o0;
        s_off1[tid] = o1;
        if (tid == 0) s_uex[BLOCK] = int32_t(utot);
        __syncthreads();
        for (uint32_t w = tid; w < utot; w += BLOCK) {
            // owner: the last list of the tile whose first unit is <= w
            int lo = 0, hi = BLOCK - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (uint32_t(s_uex[mid]) <= w) lo = mid; else hi = mid - 1;
            }
            const int local = int(w) - s_uex[lo];
            const int nc = s_nch[lo];
            const int g = nc > 0 ? local / nc : 0, ch = local - g * nc;
            const long long ib = s_off0[lo] + (long long)ch * kWarpItems;
            const long long rem = s_off1[lo] - ib;
            const int len = int(rem < kWarpItems ? rem : kWarpItems);
            const int qn = min(kQMax, s_cnt[lo] - g * kQMax);
            const long long u_idx = ubase + w;
            if (nc <= 0 || qn <= 0 || len <= 0) {
                set_error(a.err, kErrUnitDecode);
                continue;
            }
            if (u_idx < a.max_units)
                a.units[u_idx] = make_int4(int(ib), len, int(qbase + s_qex[lo] + g * kQMax), qn);
        }
        qbase += qtot;
        ubase += utot;
        __syncthreads();
    }

    // pass C: scatter the pairs whose list this CTA owns into the slot arrays
    const int npairs = a.B * a.P;
    const int W = a.W;
    for (int i = tid; i < npairs; i += BLOCK) {
        const int L = a.probe[i];
        if (L < L0 || L >= L1) continue;
        const int pos = a.list_qstart[L] + atomicAdd(&a.list_fill[L], 1);
        const int b = i / a.P;
        a.qlist[pos] = b;
        a.qmask_slot[2 * int64_t(pos)] = a.qmasks[int64_t(b) * W];
        a.qmask_slot[2 * int64_t(pos) + 1] = W > 1 ? a.qmasks[int64_t(b) * W + 1] : 0ull;
    }
}

cudaError_t launch_plan(const SearchArgs& a, int num_sms, cudaStream_t s)
{
    int G = a.nlist / 64;
    if (G > num_sms) G = num_sms;
    if (G < 1) G = 1;
    plan_kernel<kPlanBlock><<<G, kPlanBlock, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace st
