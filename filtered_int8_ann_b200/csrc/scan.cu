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
// B200 design. The plan cut the probed lists into warp units: one list chunk
// (kWarpItems rows) x up to kQMax queries probing that list, so each probed
// list is streamed once per batch whatever the number of queries probing it.
// Warps are independent (one-warp CTAs, many per SM) and take units
// round-robin, software-pipelined over three units:
//   * signature planes: the index stores each chunk's signatures as bit-planes
//     (layout.cu). A unit needs only the planes of the bits in the union of its
//     queries' masks. Each of the warp's lanes copies 16 bytes of one such
//     plane with cp.async (8 planes per warp instruction, L1 bypassed) into the
//     next free slot of a small per-warp buffer (kPlaneSlots planes); the
//     planes of the unit two ahead are requested as soon as this unit's test
//     has released its buffer. A unit whose union is wider than the buffer
//     reads its planes from global memory instead (slower, same result). Many
//     tiny copies suit the load/store path better than the bulk-copy engine,
//     whose per-request cost made 64-byte copies the bottleneck;
//   * test: for each query, the two half-warps AND the planes of the two
//     halves of the query's mask bits (a list precomputed once per search) for
//     the 32 rows of the lane's block; one shuffle joins the halves, so 32 rows
//     cost one AND per mask bit;
//   * filter-before-load: per-query survivor counts reserve candidate slots
//     (one atomic per unit and query, whose reply is needed only after the
//     survivors' rows and dots); only survivors' rows are read (16-byte
//     read-only loads) and dotted with dp4a against the query vectors (staged
//     in shared memory by cp.async while the previous unit finished); a key's
//     slot is its ballot rank among the unit's survivors of that query; each
//     key also counts into the query's score histogram, which the final top-k
//     uses to find its cut without sorting every candidate.
// cp.async groups complete in order; each unit commits exactly two groups
// (the planes two ahead, then the next unit's query vectors), so fixed
// wait_group depths find every copy: no spin loop, nothing to time out.
#include "st_internal.cuh"

namespace st {

constexpr int kPlaneSlots = 32;                         // planes one buffer holds
constexpr int kPlaneBytes = kWarpItems / 8;             // 64 bytes per plane
constexpr int kPlaneBufBytes = kPlaneSlots * kPlaneBytes;

// Per-warp shared memory: 2 plane buffers | survivor offsets [kWarpItems] u16 |
// pass words [kQMax][16] | query vectors [kQMax][d] | bit -> slot tables [2][128] |
// slot -> bit [kPlaneSlots] | query ids [kQMax]
__host__ __device__ inline size_t scan_warp_bytes(int d, int W)
{
    (void)W;
    return (2 * kPlaneBufBytes + kWarpItems * 2 + kQMax * 16 * 4 + size_t(kQMax) * d + 2 * kMaskBitsMax +
            kPlaneSlots + kQMax * 4 + 127) / 128 * 128;
}

size_t scan_smem_bytes(int d, int W) { return size_t(kScanBlock / 32) * scan_warp_bytes(d, W); }

// Request the planes a unit needs (the union u0/u1 of its queries' mask bits)
// into consecutive slots of `buf`, recording bit -> slot in `tab`. Returns
// false (and copies nothing) when the union has more bits than a buffer
// holds. The caller commits the group.
template <int W>
__device__ __forceinline__ bool issue_planes(const SearchArgs& a, int chunk, uint64_t u0, uint64_t u1,
                                             uint32_t* buf, uint8_t* tab, uint8_t* inv, int lane)
{
    constexpr int NPL = 64 * W;
    const int n0 = __popcll(u0);
    const int nb = n0 + (W > 1 ? __popcll(u1) : 0);
    if (nb > kPlaneSlots) return false;  // warp-uniform
    __syncwarp();  // earlier reads of tab / inv are done
#pragma unroll
    for (int r = 0; r < 2 * W; ++r) {
        const int b = lane + 32 * r;
        const uint64_t word = b < 64 ? u0 : u1;
        const uint64_t below = (b & 63) ? (word & ((1ull << (b & 63)) - 1ull)) : 0ull;
        const int slot = (b < 64 ? 0 : n0) + __popcll(below);
        const bool on = (word >> (b & 63)) & 1ull;
        tab[b] = on ? uint8_t(slot) : uint8_t(0);
        if (on) inv[slot] = uint8_t(b);
    }
    __syncwarp();
    // lane = 4 * (plane of this round) + (16-byte quarter of the plane)
    const uint32_t* src = a.planes + int64_t(chunk) * NPL * 16 + (lane & 3) * 4;
    for (int j = lane >> 2; j < nb; j += 8) cp_async16_cg(buf + j * 16 + (lane & 3) * 4, src + inv[j] * 16);
    return true;
}

// OR of the masks held by lanes < qn (other lanes hold zeros).
__device__ __forceinline__ void warp_or2(uint64_t& x, uint64_t& y)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        x |= __shfl_xor_sync(0xffffffffu, x, off);
        y |= __shfl_xor_sync(0xffffffffu, y, off);
    }
}

// NP = d/16 when the row is held in registers (d = 64 or 128), 0 for any other
// d (rows are then re-read from L1 for each eligible query).
// (at most as many registers as keep the shared-memory-limited warp count resident)
template <int NP, int W>
__global__ void __launch_bounds__(kScanBlock, NP == 8 ? 16 : 20)
scan_kernel(SearchArgs a)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    constexpr int NPL = 64 * W;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int d = a.d;
    const int np = NP ? NP : (d >> 4);
    const int blk = lane & 15;   // 32-row block of the chunk this lane tests
    const int half = lane >> 4;  // which half of the mask bits it ANDs

    unsigned char* wb = smem_raw + size_t(warp) * scan_warp_bytes(d, W);
    uint32_t* const pbuf0 = reinterpret_cast<uint32_t*>(wb);
    uint32_t* const pbuf1 = reinterpret_cast<uint32_t*>(wb + kPlaneBufBytes);
    uint16_t* surv = reinterpret_cast<uint16_t*>(wb + 2 * kPlaneBufBytes);              // [kWarpItems]
    uint32_t* s_pass = reinterpret_cast<uint32_t*>(surv + kWarpItems);                   // [kQMax][16]
    int4* s_q = reinterpret_cast<int4*>(s_pass + kQMax * 16);                            // [kQMax][np]
    uint8_t* s_tab = reinterpret_cast<uint8_t*>(s_q) + size_t(kQMax) * d;                // [2][128]
    uint8_t* s_inv = s_tab + 2 * kMaskBitsMax;                                           // [kPlaneSlots]
    int32_t* s_qid = reinterpret_cast<int32_t*>(s_inv + kPlaneSlots);                    // [kQMax]

    const int n_units = a.ctl->n_units < a.max_units ? a.ctl->n_units : a.max_units;
    const int stride = gridDim.x * (kScanBlock / 32);
    int u = blockIdx.x * (kScanBlock / 32) + warp;
    if (u >= n_units) return;

    // unit entry: {first row, chunk, first query slot, rows << 16 | queries}
    auto load_slots = [&](const int4& e, int& qid, uint64_t& m0, uint64_t& m1) {
        qid = 0;
        m0 = 0;
        m1 = 0;
        if (lane < (e.w & 0xFFFF)) {
            qid = a.qlist[e.z + lane];
            const ulonglong2 m = reinterpret_cast<const ulonglong2*>(a.qmask_slot)[e.z + lane];
            m0 = m.x;
            m1 = m.y;
        }
    };
    // query ids of a unit -> shared memory, its query vectors by cp.async
    auto stage_queries = [&](int qn, int qid) {
        __syncwarp();  // earlier reads of s_qid / s_q are done
        if (lane < qn) s_qid[lane] = qid;
        __syncwarp();
        for (int idx = lane; idx < qn * np; idx += 32) {
            const int s = idx / np, p = idx - s * np;
            cp_async16(s_q + s * np + p, a.queries + int64_t(s_qid[s]) * d + 16 * p);
        }
    };

    // Request the planes of a unit whose entry is `e` and whose slots (lanes <
    // its query count) hold masks m0/m1, into buffer `bb`; returns the number
    // of planes the buffer then holds, or -1 when the test must read global
    // planes. A single-query unit needs no union: its planes are the query's
    // mask bits in increasing order, listed by the probe.
    auto request_planes = [&](const int4& e, int qid, uint64_t m0, uint64_t m1, int bb) -> int {
        uint32_t* buf = bb ? pbuf1 : pbuf0;
        if ((e.w & 0xFFFF) == 1) {
            const int q = __shfl_sync(0xffffffffu, qid, 0);
            const int nb = __ldg(a.qnbits + q);
            if (nb > kPlaneSlots) return -1;
            const uint8_t* bits = a.qbits + int64_t(q) * kMaskBitsMax;
            const uint32_t* src = a.planes + int64_t(e.y) * NPL * 16 + (lane & 3) * 4;
            for (int j = lane >> 2; j < nb; j += 8)
                cp_async16_cg(buf + j * 16 + (lane & 3) * 4, src + __ldg(bits + j) * 16);
            return nb;
        }
        uint64_t x = m0, y = m1;
        warp_or2(x, y);
        if (!issue_planes<W>(a, e.y, x, y, buf, s_tab + bb * kMaskBitsMax, s_inv, lane)) return -1;
        return __popcll(x) + (W > 1 ? __popcll(y) : 0);
    };

    // prologue: entries of the first three units, slots of the first two;
    // groups: planes(0), queries(0), planes(1)
    int4 e_cur = a.units[u];
    int4 e_nxt = make_int4(0, 0, 0, 0), e_n2 = make_int4(0, 0, 0, 0);
    const bool has_nxt0 = u + stride < n_units;
    if (has_nxt0) e_nxt = a.units[u + stride];
    if (u + 2 * stride < n_units) e_n2 = a.units[u + 2 * stride];
    int qid_c, qid_n = 0;
    uint64_t m0_c, m1_c, m0_n = 0, m1_n = 0;
    load_slots(e_cur, qid_c, m0_c, m1_c);
    if (has_nxt0) load_slots(e_nxt, qid_n, m0_n, m1_n);
    int held0 = request_planes(e_cur, qid_c, m0_c, m1_c, 0);  // planes held by buffer 0 / 1 (-1: global)
    cp_async_commit();
    stage_queries(e_cur.w & 0xFFFF, qid_c);
    cp_async_commit();
    int held1 = has_nxt0 ? request_planes(e_nxt, qid_n, m0_n, m1_n, 1) : -1;
    cp_async_commit();
    int b = 0;

    for (; u < n_units; u += stride) {
        const int64_t ib = e_cur.x;
        const int chunk = e_cur.y;
        const int len = e_cur.w >> 16;
        const int qn = e_cur.w & 0xFFFF;
        const uint32_t* pb = b ? pbuf1 : pbuf0;
        const uint8_t* tab = s_tab + b * kMaskBitsMax;
        const int held = b ? held1 : held0;
        const bool in_smem = held >= 0;
        const bool single = qn == 1 && in_smem;  // warp-uniform fast path
        const bool has_n2 = u + 2 * stride < n_units;
        const bool has_n3 = u + 3 * stride < n_units;

        // background loads: the entry three units ahead, the slots of the unit
        // two ahead (whose entry arrived during the previous unit)
        int4 e_n3 = make_int4(0, 0, 0, 0);
        if (has_n3) e_n3 = a.units[u + 3 * stride];
        int qid_2 = 0;
        uint64_t m0_2 = 0, m1_2 = 0;
        if (has_n2) load_slots(e_n2, qid_2, m0_2, m1_2);

        // this unit's planes: pending groups are at most [queries(u), planes(u+1)]
        cp_async_wait_group<2>();
        __syncwarp();

        // test: pass word of query s for block `blk` = AND of its mask planes;
        // the two half-warps AND the two halves of the query's mask bits
        const uint32_t valid = len >= 32 * (blk + 1) ? 0xFFFFFFFFu
                             : (len <= 32 * blk ? 0u : ((1u << (len - 32 * blk)) - 1u));
        uint32_t any = 0;
        uint32_t mycnt = 0;  // lane s: survivors of query s
        if (single) {
            // the buffer holds exactly the query's planes, in bit order
            const int h0 = (held + 1) >> 1;
            const int j1 = half ? held : h0;
            int j = half ? h0 : 0;
            uint32_t acc = 0xFFFFFFFFu;
            for (; j + 4 <= j1; j += 4)
                acc &= pb[j * 16 + blk] & pb[(j + 1) * 16 + blk] & pb[(j + 2) * 16 + blk] & pb[(j + 3) * 16 + blk];
            for (; j < j1; ++j) acc &= pb[j * 16 + blk];
            acc &= __shfl_xor_sync(0xffffffffu, acc, 16);
            any = acc & valid;
        } else {
            const uint32_t* gpl = a.planes + int64_t(chunk) * NPL * 16 + blk;
            for (int s = 0; s < qn; ++s) {
                const int qg = s_qid[s];
                const int nb = __ldg(a.qnbits + qg);
                const int h0 = (nb + 1) >> 1;
                const uint8_t* bits = a.qbits + int64_t(qg) * kMaskBitsMax;
                const int j0 = half ? h0 : 0, j1 = half ? nb : h0;
                // four independent bit -> slot -> plane chains per step
                uint32_t acc = 0xFFFFFFFFu;
                if (in_smem) {
                    int j = j0;
                    for (; j + 4 <= j1; j += 4) {
                        const int b0 = __ldg(bits + j), b1 = __ldg(bits + j + 1);
                        const int b2 = __ldg(bits + j + 2), b3 = __ldg(bits + j + 3);
                        const int s0 = tab[b0], s1 = tab[b1], s2 = tab[b2], s3 = tab[b3];
                        acc &= pb[s0 * 16 + blk] & pb[s1 * 16 + blk] & pb[s2 * 16 + blk] & pb[s3 * 16 + blk];
                    }
                    for (; j < j1; ++j) acc &= pb[tab[__ldg(bits + j)] * 16 + blk];
                } else {
                    for (int j = j0; j < j1; ++j) acc &= __ldg(gpl + __ldg(bits + j) * 16);
                }
                acc &= __shfl_xor_sync(0xffffffffu, acc, 16);
                acc &= valid;
                if (half == 0) s_pass[s * 16 + blk] = acc;
                any |= acc;
                // survivors of query s: half 0 holds the 16 pass words; the full
                // 32-lane reduction leaves the total in every lane
                uint32_t c = half == 0 ? uint32_t(__popc(acc)) : 0u;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
                if (lane == s) mycnt = c;
            }
        }

        // buffer b is free: request the planes of the unit two ahead
        if (has_n2) {
            __syncwarp();  // every lane is done reading buffer b
            const int h2 = request_planes(e_n2, qid_2, m0_2, m1_2, b);
            if (b) held1 = h2;
            else held0 = h2;
        }
        cp_async_commit();

        // survivor row offsets, block by block
        const uint32_t mine = half == 0 ? uint32_t(__popc(any)) : 0u;
        uint32_t incl = mine;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += t;
        }
        const int nsurv = int(__shfl_sync(0xffffffffu, incl, 31));
        if (half == 0) {
            int pos = int(incl - mine);
            uint32_t rest = any;
            while (rest) {
                const int i = __ffs(rest) - 1;
                rest &= rest - 1u;
                surv[pos++] = uint16_t(32 * blk + i);
            }
        }

        // per-query survivor counts -> one reservation each (lane s); the
        // reply is first needed when the keys are stored
        if (single && lane == 0) mycnt = uint32_t(nsurv);
        uint32_t base = 0;
        if (lane < qn && mycnt) {
            base = atomicAdd(&a.cand_cnt[int64_t(qid_c) * kCntStride], mycnt);
            atomicAdd(&a.eligible_cnt[int64_t(qid_c) * (kCntStride / 2)], (unsigned long long)mycnt);
        }

        // this unit's query vectors: pending groups are at most [planes(u+2)]
        cp_async_wait_group<1>();
        __syncwarp();

        // rows of the survivors (one load per survivor), dots, keys into the
        // reserved slots
        if (single) {
            // every survivor is a key of the one query, in survivor order
            const int qg = s_qid[0];
            uint64_t* cand = a.cand + int64_t(qg) * a.cap;
            uint32_t* hist = a.hist + int64_t(qg) * kHistBins;
            for (int c0 = 0; c0 < nsurv; c0 += 32) {
                const int idx = c0 + lane;
                int4 row[NP > 0 ? NP : 1];
                const int4* rp = nullptr;
                int64_t i = 0;
                if (idx < nsurv) {
                    i = ib + surv[idx];
                    rp = reinterpret_cast<const int4*>(a.items + i * d);
                    if (NP > 0) {
#pragma unroll
                        for (int p = 0; p < (NP > 0 ? NP : 1); ++p) row[p] = __ldg(rp + p);
                    }
                }
                const uint32_t base0 = __shfl_sync(0xffffffffu, base, 0);
                if (idx < nsurv) {
                    int32_t acc0 = 0, acc1 = 0;
                    if (NP > 0) {
#pragma unroll
                        for (int p = 0; p < (NP > 0 ? NP : 1); p += 2) {
                            acc0 = dot16(row[p], s_q[p], acc0);
                            if (p + 1 < NP) acc1 = dot16(row[p + 1], s_q[p + 1], acc1);
                        }
                    } else {
                        for (int p = 0; p < np; ++p) acc0 = dot16(__ldg(rp + p), s_q[p], acc0);
                    }
                    const int32_t score = acc0 + acc1;
                    const uint64_t pos = uint64_t(base0) + uint32_t(idx);
                    if (pos < uint64_t(a.cap)) cand[pos] = pack_key(score, uint32_t(i));
                    atomicAdd(&hist[score_bin(score, a.smax, a.hshift)], 1u);
                }
            }
        } else {
            // a key's slot is its ballot rank among this unit's survivors of
            // the same query
            uint32_t run = 0;  // lane s: keys of query s written so far
            for (int c0 = 0; c0 < nsurv; c0 += 32) {
                const int idx = c0 + lane;
                int off = -1;
                int64_t i = 0;
                int4 row[NP > 0 ? NP : 1];
                const int4* rp = nullptr;
                if (idx < nsurv) {
                    off = surv[idx];
                    i = ib + off;
                    rp = reinterpret_cast<const int4*>(a.items + i * d);
                    if (NP > 0) {
#pragma unroll
                        for (int p = 0; p < (NP > 0 ? NP : 1); ++p) row[p] = __ldg(rp + p);
                    }
                }
                const uint32_t* pw = s_pass + (off >= 0 ? (off >> 5) : 0);
                const int bit = off & 31;
                for (int s = 0; s < qn; ++s) {
                    const bool on = off >= 0 && ((pw[s * 16] >> bit) & 1u);
                    const unsigned bal = __ballot_sync(0xffffffffu, on);
                    if (bal == 0u) continue;
                    const uint32_t slot0 = __shfl_sync(0xffffffffu, base, s) + __shfl_sync(0xffffffffu, run, s);
                    if (on) {
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
                        const int32_t score = acc0 + acc1;
                        const int qg = s_qid[s];
                        if (pos < uint64_t(a.cap)) a.cand[int64_t(qg) * a.cap + int64_t(pos)] = pack_key(score, uint32_t(i));
                        atomicAdd(&a.hist[int64_t(qg) * kHistBins + score_bin(score, a.smax, a.hshift)], 1u);
                    }
                    if (lane == s) run += __popc(bal);
                }
            }
        }

        // the next unit's query vectors (group queries(u+1))
        stage_queries(e_nxt.w & 0xFFFF, qid_n);
        cp_async_commit();

        e_cur = e_nxt;
        e_nxt = e_n2;
        e_n2 = e_n3;
        qid_c = qid_n;
        m0_c = m0_n;
        m1_c = m1_n;
        qid_n = qid_2;
        m0_n = m0_2;
        m1_n = m1_2;
        b ^= 1;
    }
    cp_async_wait_all();  // no copy may land after the warp has left
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
