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
// B200 design. The plan kernel cut the probed lists into warp units (up to
// kWarpItems consecutive rows x up to kQMax queries probing that list), so each
// probed list is streamed once per batch whatever the number of queries
// probing it. Warps are independent and take units round-robin; each warp runs
// a two-stage software pipeline:
//   * signatures: the unit's contiguous signature block (16 B per row for
//     128-bit signatures) arrives by one bulk asynchronous copy (TMA engine,
//     cp.async.bulk + mbarrier) into one of two per-warp shared buffers; the
//     copy for the next unit is always in flight while this one is processed,
//     so the signature stream never waits on the rest of the pipeline;
//   * test: every signature against every query of the unit (masks by warp
//     shuffle) gives a per-row query bitmask; the per-query survivor counts
//     reserve candidate slots with one atomic per (unit, query), issued before
//     the row loads so both round trips overlap;
//   * filter-before-load: only survivors' rows are read (16-byte read-only
//     loads into registers) -- rows of ineligible items never leave HBM -- and
//     dotted with dp4a against the query vectors (staged in shared memory by
//     cp.async); keys go straight to the reserved slots.
// Every wait on a copy is bounded: on expiry the warp records kErrCopyTimeout,
// waits (bounded) for its copies in flight and stops.
#include "st_internal.cuh"

namespace st {

template <int W>
struct SigBuf {
    // bytes of one signature buffer: a unit's signatures plus 16 bytes so that
    // a 64-bit-signature copy can start at the 16-byte boundary below its row
    static constexpr int kBytes = ((kWarpItems * 8 * W + 16) + 127) / 128 * 128;
};

__host__ __device__ inline size_t scan_warp_bytes(int d, int W)
{
    const size_t sig = W == 2 ? SigBuf<2>::kBytes : SigBuf<1>::kBytes;
    // 2 signature buffers | query vectors [kQMax][d] | masks [kQMax][2] | qid [kQMax] | 2 mbarriers
    return (2 * sig + size_t(kQMax) * d + kQMax * 16 + kQMax * 4 + 16 + 127) / 128 * 128;
}

size_t scan_smem_bytes(int d, int W) { return size_t(kScanBlock / 32) * scan_warp_bytes(d, W); }

template <int W>
__device__ __forceinline__ void issue_sig_copy(const SearchArgs& a, int4 e, unsigned char* buf, uint64_t* bar)
{
    const int64_t ib = e.x;
    const int len = e.y;
    const char* src;
    uint32_t bytes;
    if (W == 2) {
        src = reinterpret_cast<const char*>(a.sigs + ib * 2);
        bytes = uint32_t(len) * 16u;
    } else {
        const int64_t a0 = ib & ~int64_t(1);
        src = reinterpret_cast<const char*>(a.sigs + a0);
        bytes = uint32_t(((ib + len - a0) * 8 + 15) & ~int64_t(15));
    }
    mbar_expect_tx(bar, bytes);
    bulk_g2s(buf, src, bytes, bar);
}

// NP = d/16 when the row is held in registers (d = 64 or 128), 0 for any other
// d (rows are then re-read from L1 for each eligible query).
template <int NP, int W>
__global__ void __launch_bounds__(kScanBlock)
scan_kernel(SearchArgs a)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    constexpr int IPL = kWarpItems / 32;  // rows per lane
    constexpr int SB = SigBuf<W>::kBytes;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int d = a.d;
    const int np = NP ? NP : (d >> 4);

    unsigned char* wb = smem_raw + size_t(warp) * scan_warp_bytes(d, W);
    unsigned char* sbuf0 = wb;
    unsigned char* sbuf1 = wb + SB;
    int4* s_q = reinterpret_cast<int4*>(wb + 2 * SB);                                // [kQMax][np]
    ulonglong2* s_m = reinterpret_cast<ulonglong2*>(wb + 2 * SB + size_t(kQMax) * d); // [kQMax]
    int32_t* s_qid = reinterpret_cast<int32_t*>(s_m + kQMax);                         // [kQMax]
    uint64_t* bars = reinterpret_cast<uint64_t*>(s_qid + kQMax);                      // [2]

    if (lane == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
    }
    __syncwarp();

    const int n_units = a.ctl->n_units;
    const int stride = gridDim.x * (kScanBlock / 32);
    int u = blockIdx.x * (kScanBlock / 32) + warp;
    if (u >= n_units) return;

    // prologue: copies for the first two units, slots of the first
    int4 e_cur = a.units[u];
    int4 e_nxt = make_int4(0, 0, 0, 0);
    const bool has_nxt0 = u + stride < n_units;
    if (has_nxt0) e_nxt = a.units[u + stride];
    if (lane == 0) {
        issue_sig_copy<W>(a, e_cur, sbuf0, &bars[0]);
        if (has_nxt0) issue_sig_copy<W>(a, e_nxt, sbuf1, &bars[1]);
    }
    int qid_c = 0;
    uint64_t m0_c = 0, m1_c = 0;
    if (lane < e_cur.w) {
        qid_c = a.qlist[e_cur.z + lane];
        m0_c = a.qmask_slot[2 * int64_t(e_cur.z + lane)];
        m1_c = a.qmask_slot[2 * int64_t(e_cur.z + lane) + 1];
    }
    uint32_t phase = 0;   // bit b: parity to wait for on buffer b
    uint32_t pending = has_nxt0 ? 3u : 1u;  // bit b: a copy into buffer b is in flight
    int b = 0;

    for (; u < n_units; u += stride) {
        const int64_t ib = e_cur.x;
        const int len = e_cur.y;
        const int qn = e_cur.w;
        unsigned char* sb = b ? sbuf1 : sbuf0;
        const bool has_nxt = u + stride < n_units;
        const bool has_n2 = u + 2 * stride < n_units;

        // background loads for later units: entry two ahead, slots one ahead
        int4 e_n2 = make_int4(0, 0, 0, 0);
        if (has_n2) e_n2 = a.units[u + 2 * stride];
        int qid_n = 0;
        uint64_t m0_n = 0, m1_n = 0;
        if (has_nxt && lane < e_nxt.w) {
            qid_n = a.qlist[e_nxt.z + lane];
            m0_n = a.qmask_slot[2 * int64_t(e_nxt.z + lane)];
            m1_n = a.qmask_slot[2 * int64_t(e_nxt.z + lane) + 1];
        }

        // query ids and masks of this unit -> shared memory; vectors by cp.async
        if (lane < qn) {
            s_qid[lane] = qid_c;
            s_m[lane] = make_ulonglong2(m0_c, m1_c);
        }
        __syncwarp();
        for (int idx = lane; idx < qn * np; idx += 32) {
            const int s = idx / np, p = idx - s * np;
            cp_async16(s_q + s * np + p, a.queries + int64_t(s_qid[s]) * d + 16 * p);
        }
        cp_async_commit();

        // wait for this unit's signatures
        const bool ok = mbar_wait_bounded(&bars[b], (phase >> b) & 1u);
        if (!__all_sync(0xffffffffu, ok)) {
            if (lane == 0) set_error(a.err, kErrCopyTimeout);
            break;
        }
        phase ^= 1u << b;
        pending &= ~(1u << b);

        // test every row against every query of the unit: bit s of em[j] is set
        // when row lane+32j carries every bit of query s's mask
        uint32_t em[IPL];
        const int off1 = (W == 1) ? int(ib & 1) : 0;
#pragma unroll
        for (int j = 0; j < IPL; ++j) {
            const int t = lane + 32 * j;
            uint32_t e = 0;
            if (t < len) {
                if (W == 2) {
                    const ulonglong2 v = reinterpret_cast<const ulonglong2*>(sb)[t];
                    for (int s = 0; s < qn; ++s) {
                        const ulonglong2 m = s_m[s];
                        const uint64_t miss = (~v.x & m.x) | (~v.y & m.y);
                        e |= uint32_t(miss == 0ull) << s;
                    }
                } else {
                    const uint64_t v = reinterpret_cast<const uint64_t*>(sb)[off1 + t];
                    for (int s = 0; s < qn; ++s) {
                        const uint64_t m = s_m[s].x;
                        e |= uint32_t((~v & m) == 0ull) << s;
                    }
                }
            }
            em[j] = e;
        }

        // compact the survivors into this unit's (now consumed) signature buffer
        __syncwarp();
        uint64_t* surv = reinterpret_cast<uint64_t*>(sb);
        int nsurv = 0;
#pragma unroll
        for (int j = 0; j < IPL; ++j) {
            const unsigned bal = __ballot_sync(0xffffffffu, em[j] != 0u);
            if (em[j]) surv[nsurv + __popc(bal & lanemask_lt())] = (uint64_t(lane + 32 * j) << 32) | em[j];
            nsurv += __popc(bal);
        }
        cp_async_wait_all();
        __syncwarp();

        // survivors per query (lane s counts query s) -> one reservation each
        uint32_t mycnt = 0;
        for (int c0 = 0; c0 < nsurv; c0 += 32) {
            const uint32_t e = (c0 + lane < nsurv) ? uint32_t(surv[c0 + lane]) : 0u;
            for (int s = 0; s < qn; ++s) {
                const uint32_t ns = __popc(__ballot_sync(0xffffffffu, (e >> s) & 1u));
                if (lane == s) mycnt += ns;
            }
        }
        uint32_t base = 0;
        if (lane < qn && mycnt) {
            base = atomicAdd(&a.cand_cnt[qid_c], mycnt);
            atomicAdd(&a.eligible_cnt[qid_c], (unsigned long long)mycnt);
        }

        // rows of the survivors (one load per survivor), dots, keys into the
        // reserved slots; a key's slot is its rank among this unit's survivors
        // of the same query (ballot prefix), so no shared atomics are needed
        uint32_t run = 0;  // lane s: keys of query s written so far
        for (int c0 = 0; c0 < nsurv; c0 += 32) {
            const int idx = c0 + lane;
            uint32_t e = 0;
            int64_t i = 0;
            int4 row[NP > 0 ? NP : 1];
            const int4* rp = nullptr;
            if (idx < nsurv) {
                const uint64_t sv = surv[idx];
                e = uint32_t(sv);
                i = ib + int64_t(sv >> 32);
                rp = reinterpret_cast<const int4*>(a.items + i * d);
                if (NP > 0) {
#pragma unroll
                    for (int p = 0; p < (NP > 0 ? NP : 1); ++p) row[p] = __ldg(rp + p);
                }
            }
            for (int s = 0; s < qn; ++s) {
                const bool mine = (e >> s) & 1u;
                const unsigned bal = __ballot_sync(0xffffffffu, mine);
                if (bal == 0u) continue;
                const uint32_t slot0 = __shfl_sync(0xffffffffu, base, s) + __shfl_sync(0xffffffffu, run, s);
                if (mine) {
                    const int4* qs = s_q + s * np;
                    int32_t acc0 = 0, acc1 = 0;
                    if (NP > 0) {
#pragma unroll
                        for (int p = 0; p < (NP > 0 ? NP : 1); p += 2) {
                            acc0 = dot16(row[p], qs[p], acc0);
                            if (p + 1 < NP) acc1 = dot16(row[p + 1], qs[p + 1], acc1);
                        }
                    } else {
                        for (int p = 0; p < np; ++p) acc0 = dot16(__ldg(rp + p), qs[p], acc0);
                    }
                    const uint64_t pos = uint64_t(slot0) + __popc(bal & lanemask_lt());
                    if (pos < uint64_t(a.cap))
                        a.cand[int64_t(s_qid[s]) * a.cap + int64_t(pos)] = pack_key(acc0 + acc1, uint32_t(i));
                }
                if (lane == s) run += __popc(bal);
            }
        }
        fence_proxy_async_smem();
        __syncwarp();

        // buffer b is free: start the copy for the unit two ahead
        if (has_n2 && lane == 0) issue_sig_copy<W>(a, e_n2, sb, &bars[b]);
        if (has_n2) pending |= 1u << b;
        e_cur = e_nxt;
        e_nxt = e_n2;
        qid_c = qid_n;
        m0_c = m0_n;
        m1_c = m1_n;
        b ^= 1;
    }

    // after an error exit: let copies still in flight land before the warp
    // leaves (bounded)
    for (int bb = 0; bb < 2; ++bb)
        if ((pending >> bb) & 1u) mbar_wait_bounded(&bars[bb], (phase >> bb) & 1u);
    cp_async_wait_all();
}

template <int NP, int W>
static cudaError_t launch_variant(const SearchArgs& a, int num_sms, cudaStream_t s)
{
    const size_t smem = scan_smem_bytes(a.d, W);
    const void* fn = reinterpret_cast<const void*>(scan_kernel<NP, W>);
    const int slot = 1 + (NP == 4 ? 0 : NP == 8 ? 1 : 2) + 3 * (W - 1);
    cudaError_t e = ensure_smem_attr(fn, slot, int(scan_smem_bytes(ST_MAX_D, W)));
    if (e != cudaSuccess) return e;
    // occupancy depends on d only through the shared memory size: cache it for
    // the fixed-d variants
    static int occ_cache[64][8] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    int occ = (NP > 0 && dev < 64) ? occ_cache[dev][slot - 1] : 0;
    if (occ == 0) {
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, scan_kernel<NP, W>, kScanBlock, smem);
        if (e != cudaSuccess) return e;
        if (occ < 1) occ = 1;
        if (NP > 0 && dev < 64) occ_cache[dev][slot - 1] = occ;
    }
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
