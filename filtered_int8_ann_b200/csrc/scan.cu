// Fused list scan: Bloom eligibility test -> int8 inner product of the
// survivors -> candidate keys, in one pass over each probed list.
//
// The method (SilverTorch: Index as Model, section on redesigning each stage as
// a pure PyTorch module): every item carries a compact Bloom signature tested
// with one bit operation against the request mask (Bloom index filter
// paragraph); only the items that pass are scored, by an int8 inner product
// (fused Int8 ANN paragraph); the filter runs only inside the probed clusters
// (section on how each component worked before). The Andromeda review (Meta
// Andromeda, section on why the bottleneck moved from compute to bandwidth)
// gives the fusion principle kept here: intermediates stay in registers and
// shared memory and never round-trip through HBM.
//
// B200 design. Work is split into warp-sized units: up to kWarpItems
// consecutive rows of one probed list and a group of up to kQMax queries
// probing that list (built by the plan kernels), so each probed list is
// streamed once per batch whatever the number of queries probing it. Warps
// are independent: each pulls units from a device counter (prefetching the next
// unit id while it works) and never waits on the rest of its CTA, so the many
// resident warps of an SM overlap each other's memory latency.
//   1. Signatures: each lane issues all kWarpItems/32 coalesced 16-byte (or
//      8-byte) loads of its items before testing any; the query masks come in
//      by warp shuffles. Each signature is tested against every query of the
//      group into a per-item query bitmask.
//   2. Filter-before-load: items eligible for at least one query are compacted
//      (ballot + popc) into a per-warp survivor list in shared memory, and only
//      their rows are read -- rows of ineligible items never leave HBM.
//   3. Survivor rows are read with 16-byte read-only loads into registers and
//      dotted with dp4a against each eligible query's vector (shared memory).
//   4. Keys (score, id) are appended to per-query candidate buffers with one
//      global atomic per (warp, query) group (match_any aggregation).
#include "st_internal.cuh"

namespace st {

__device__ __forceinline__ void warp_append(bool emit, int q, uint64_t key, const SearchArgs& a)
{
    const unsigned act = __ballot_sync(0xffffffffu, emit);
    if (act == 0u || !emit) return;
    const unsigned peers = __match_any_sync(act, q);
    const int leader = __ffs(peers) - 1;
    const int lane = threadIdx.x & 31;
    uint32_t base = 0;
    if (lane == leader) base = atomicAdd(&a.cand_cnt[q], uint32_t(__popc(peers)));
    base = __shfl_sync(peers, base, leader);
    const uint64_t pos = uint64_t(base) + uint64_t(__popc(peers & lanemask_lt()));
    if (pos < uint64_t(a.cap)) a.cand[int64_t(q) * a.cap + int64_t(pos)] = key;
}

template <int W>
struct SigT;
template <>
struct SigT<1> {
    uint64_t w0;
    __device__ __forceinline__ void load(const uint64_t* p) { w0 = __ldg(p); }
    __device__ __forceinline__ bool pass(uint64_t m0, uint64_t) const { return (w0 & m0) == m0; }
};
template <>
struct SigT<2> {
    uint64_t w0, w1;
    __device__ __forceinline__ void load(const uint64_t* p)
    {
        const ulonglong2 v = __ldg(reinterpret_cast<const ulonglong2*>(p));
        w0 = v.x;
        w1 = v.y;
    }
    __device__ __forceinline__ bool pass(uint64_t m0, uint64_t m1) const
    {
        return ((w0 & m0) == m0) & ((w1 & m1) == m1);
    }
};

// Per-warp shared memory: query vectors [kQMax][d], query ids, survivors,
// per-query eligible counts.
struct WarpSmemLayout {
    static __host__ __device__ size_t bytes(int d)
    {
        return size_t(kQMax) * d + kQMax * 4 + kQMax * 4 + kWarpItems * 8;
    }
};

// NP = d/16 when the row is held in registers (d = 64 or 128), 0 for any other
// d (rows are then re-read from L1 for each eligible query).
template <int NP, int W>
__global__ void __launch_bounds__(kScanBlock)
scan_kernel(SearchArgs a)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    constexpr int IPL = kWarpItems / 32;  // items per lane
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int d = a.d;
    const int np = NP ? NP : (d >> 4);

    unsigned char* wbase = smem_raw + size_t(warp) * WarpSmemLayout::bytes(d);
    int4* s_q = reinterpret_cast<int4*>(wbase);                                  // [kQMax][np]
    int32_t* s_qid = reinterpret_cast<int32_t*>(wbase + size_t(kQMax) * d);       // [kQMax]
    uint32_t* s_elig = reinterpret_cast<uint32_t*>(s_qid + kQMax);                 // [kQMax]
    uint64_t* s_surv = reinterpret_cast<uint64_t*>(s_elig + kQMax);                // [kWarpItems]

    const int n_units = a.ctl->n_units;
    int u = 0;
    if (lane == 0) u = atomicAdd(&a.ctl->next_unit, 1);
    u = __shfl_sync(0xffffffffu, u, 0);

    while (u < n_units) {
        const int4 e = a.units[u];
        const int64_t ib = e.x;
        const int len = e.y, qoff = e.z, qn = e.w;
        int un = 0;
        if (lane == 0) un = atomicAdd(&a.ctl->next_unit, 1);  // prefetch the next unit id

        // 1. signature loads, all in flight together
        SigT<W> sg[IPL];
#pragma unroll
        for (int j = 0; j < IPL; ++j)
            if (lane + 32 * j < len) sg[j].load(a.sigs + (ib + lane + 32 * j) * W);

        // query ids and masks of the group (lane s holds query s)
        int qid = 0;
        uint64_t m0 = 0, m1 = 0;
        if (lane < qn) {
            qid = a.qlist[qoff + lane];
            const uint64_t* mp = a.qmasks + int64_t(qid) * W;
            m0 = mp[0];
            if (W > 1) m1 = mp[W - 1];
            s_qid[lane] = qid;
            s_elig[lane] = 0;
        }
        __syncwarp();
        for (int idx = lane; idx < qn * np; idx += 32) {
            const int s = idx / np, p = idx - s * np;
            s_q[s * np + p] = reinterpret_cast<const int4*>(a.queries + int64_t(s_qid[s]) * d)[p];
        }

        // 2. test every item against every query of the group
        uint32_t em[IPL];
#pragma unroll
        for (int j = 0; j < IPL; ++j) em[j] = 0;
        for (int s = 0; s < qn; ++s) {
            const uint64_t q0 = __shfl_sync(0xffffffffu, m0, s);
            const uint64_t q1 = __shfl_sync(0xffffffffu, m1, s);
#pragma unroll
            for (int j = 0; j < IPL; ++j)
                if (lane + 32 * j < len && sg[j].pass(q0, q1)) em[j] |= 1u << s;
        }
        int nsurv = 0;
#pragma unroll
        for (int j = 0; j < IPL; ++j) {
            const unsigned bal = __ballot_sync(0xffffffffu, em[j] != 0u);
            if (em[j]) s_surv[nsurv + __popc(bal & lanemask_lt())] = (uint64_t(lane + 32 * j) << 32) | em[j];
            nsurv += __popc(bal);
        }
        __syncwarp();

        // 3-4. survivors: rows, dots, keys
        for (int base = 0; base < nsurv; base += 32) {
            const int idx = base + lane;
            uint32_t emk = 0;
            int64_t i = 0;
            int4 row[NP > 0 ? NP : 1];
            const int4* rp = nullptr;
            if (idx < nsurv) {
                const uint64_t sv = s_surv[idx];
                emk = uint32_t(sv);
                i = ib + int64_t(sv >> 32);
                rp = reinterpret_cast<const int4*>(a.items + i * d);
                if (NP > 0) {
#pragma unroll
                    for (int p = 0; p < (NP > 0 ? NP : 1); ++p) row[p] = __ldg(rp + p);
                }
            }
            while (__any_sync(0xffffffffu, emk != 0u)) {
                bool emit = false;
                uint64_t key = 0;
                int q = 0;
                if (emk) {
                    const int s = __ffs(emk) - 1;
                    emk &= emk - 1u;
                    int32_t acc = 0;
                    const int4* qs = s_q + s * np;
                    if (NP > 0) {
#pragma unroll
                        for (int p = 0; p < (NP > 0 ? NP : 1); ++p) acc = dot16(row[p], qs[p], acc);
                    } else {
                        for (int p = 0; p < np; ++p) acc = dot16(__ldg(rp + p), qs[p], acc);
                    }
                    key = pack_key(acc, uint32_t(i));
                    q = s_qid[s];
                    emit = true;
                    atomicAdd(&s_elig[s], 1u);
                }
                warp_append(emit, q, key, a);
            }
        }
        __syncwarp();
        if (lane < qn && s_elig[lane])
            atomicAdd(&a.eligible_cnt[qid], (unsigned long long)s_elig[lane]);
        __syncwarp();
        u = __shfl_sync(0xffffffffu, un, 0);
    }
}

size_t scan_smem_bytes(int d)
{
    return size_t(kScanBlock / 32) * WarpSmemLayout::bytes(d);
}

template <int NP, int W>
static cudaError_t launch_variant(const SearchArgs& a, int num_sms, cudaStream_t s)
{
    const size_t smem = scan_smem_bytes(a.d);
    const void* fn = reinterpret_cast<const void*>(scan_kernel<NP, W>);
    cudaError_t e = ensure_smem_attr(fn, 1 + (NP == 4 ? 0 : NP == 8 ? 1 : 2) + 3 * (W - 1));
    if (e != cudaSuccess) return e;
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, scan_kernel<NP, W>, kScanBlock, smem);
    if (e != cudaSuccess) return e;
    if (occ < 1) occ = 1;
    scan_kernel<NP, W><<<num_sms * occ, kScanBlock, smem, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_scan(const SearchArgs& a, int num_sms, cudaStream_t s)
{
    if (a.W == 2) {
        if (a.d == 64) return launch_variant<4, 2>(a, num_sms, s);
        if (a.d == 128) return launch_variant<8, 2>(a, num_sms, s);
        return launch_variant<0, 2>(a, num_sms, s);
    }
    if (a.d == 64) return launch_variant<4, 1>(a, num_sms, s);
    if (a.d == 128) return launch_variant<8, 1>(a, num_sms, s);
    return launch_variant<0, 1>(a, num_sms, s);
}

}  // namespace st
