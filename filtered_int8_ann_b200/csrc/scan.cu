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
// Warps work independently (four per CTA, sharing only a unit counter) and
// take units in turn. A warp tests one unit ahead of the one it scores, so every
// memory round trip of a unit overlaps the previous unit's work:
//   * signature planes: the index stores each chunk's signatures as bit-planes
//     (layout.cu). A unit needs only the planes of the bits in the union of its
//     queries' masks (for a single-query unit: the query's own mask bits, in
//     order). Each lane copies 16 bytes of one such plane with cp.async (8
//     planes per warp instruction, L1 bypassed) into the next slot of the
//     warp's plane buffer (kPlaneSlots planes); the next unit's planes are
//     requested as soon as this unit's test has released the buffer. A unit
//     whose union is wider than the buffer reads its planes from global
//     memory instead (slower, same result);
//   * test: for each query, the two half-warps AND the planes of the two
//     halves of the query's mask bits for the 32 rows of the lane's block; one
//     shuffle joins the halves, so 32 rows cost one AND per mask bit;
//   * filter-before-load: per-query survivor counts reserve candidate slots
//     (one atomic per unit and query, answered while the previous unit is
//     scored); the first survivors' rows are copied into the warp's shared
//     memory by cp.async and the next ones prefetched into L2, so one
//     iteration later only those rows are read (from shared memory, or by
//     16-byte read-only loads) and dotted with dp4a against the query vectors
//     (staged in shared memory by cp.async); a
//     key's slot is its rank among the unit's survivors of that query, and
//     the key is counted in the query's score bins (kTcBins bins over the
//     query's possible range [-S, S]), which guide the final top-k and the
//     dense scan's running bound (not with deletions or exclude masks: this
//     scan writes the keys those drop, and the final top-k filters them).
// Every unit commits exactly two cp.async groups (planes of the unit two
// ahead, then query vectors and staged rows of the next unit), so fixed
// wait_group depths find every copy: there is no spin loop and nothing to
// time out.
#include "st_internal.cuh"

namespace st {

constexpr int kPlaneSlots = 32;                         // planes one buffer holds
static_assert(kPlaneSlots <= kSlotBits, "a slot carries every bit of a mask whose planes fit the buffer");
constexpr int kPlaneBytes = kWarpItems / 8;             // 64 bytes per plane
constexpr int kPlaneBufBytes = kPlaneSlots * kPlaneBytes;

// Survivor rows a unit stages in shared memory (its first survivors; the
// others are read from global memory): sized so that the warps the registers
// allow stay resident (five CTAs per SM for d = 64, four for d = 128).
__host__ __device__ constexpr int scan_stage_rows(int d) { return d == 64 ? 24 : d == 128 ? 16 : 0; }

// Per-warp shared memory: staged survivor rows [2][scan_stage_rows(d)][d] |
// plane buffer | survivor offsets [2][kWarpItems] u16 | pass words
// [2][kQMax][16] | query vectors [kQMax][d] | bit -> slot table [128] | slot
// -> bit [kPlaneSlots]
__host__ __device__ inline size_t scan_warp_bytes(int d, int W)
{
    (void)W;
    return (size_t(2) * scan_stage_rows(d) * d + kPlaneBufBytes + 2 * kWarpItems * 2 + 2 * kQMax * 16 * 4 +
            size_t(kQMax) * d + kMaskBitsMax + kPlaneSlots + 127) / 128 * 128;
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

// L2 prefetch of a row (one per 32-byte sector)
__device__ __forceinline__ void prefetch_l2(const void* p)
{
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// NP = d/16 when the row is held in registers (d = 64 or 128), 0 for any other
// d (rows are then re-read from L1 for each eligible query).
// (at most as many registers as keep the shared-memory-limited warp count resident)
template <int NP, int W>
__global__ void __launch_bounds__(kScanBlock, NP == 8 ? 4 : 5)
scan_kernel(SearchArgs a)
{
    dep_enter();
    extern __shared__ __align__(128) unsigned char smem_raw[];
    constexpr int NPL = 64 * W;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int d = a.d;
    const int np = NP ? NP : (d >> 4);
    const int blk = lane & 15;   // 32-row block of the chunk this lane tests
    const int half = lane >> 4;  // which half of the mask bits it ANDs

    constexpr int R = scan_stage_rows(NP * 16);  // staged rows per unit (0: none)
    unsigned char* wb = smem_raw + size_t(warp) * scan_warp_bytes(d, W);
    int4* const srow2 = reinterpret_cast<int4*>(wb);  // [2][R][NP]
    wb += size_t(2) * R * NP * 16;
    uint32_t* const pbuf = reinterpret_cast<uint32_t*>(wb);
    uint16_t* const surv2 = reinterpret_cast<uint16_t*>(wb + kPlaneBufBytes);            // [2][kWarpItems]
    uint32_t* const pass2 = reinterpret_cast<uint32_t*>(surv2 + 2 * kWarpItems);         // [2][kQMax][16]
    int4* const s_q = reinterpret_cast<int4*>(pass2 + 2 * kQMax * 16);                  // [kQMax][np]
    uint8_t* const s_tab = reinterpret_cast<uint8_t*>(s_q) + size_t(kQMax) * d;           // [128]
    uint8_t* const s_inv = s_tab + kMaskBitsMax;                                         // [kPlaneSlots]

    // units: CTA c owns units c, c + ncta, c + 2 ncta, ... (an even mix of the
    // table); its warps take them in turn from a shared counter, three units
    // ahead, so a warp that drew cheap units takes more of them
    __shared__ int s_next;
    if (threadIdx.x == 0) s_next = 0;
    __syncthreads();
    const int n_units = a.ctl->n_units < a.max_units ? a.ctl->n_units : a.max_units;
    auto draw = [&]() -> int {
        int j = 0;
        if (lane == 0) j = atomicAdd(&s_next, 1);
        j = __shfl_sync(0xffffffffu, j, 0);
        const int64_t v = int64_t(blockIdx.x) + int64_t(j) * gridDim.x;
        return v < n_units ? int(v) : n_units;
    };
    int u = draw();
    if (u >= n_units) return;
    // keys are counted in the score bins only when every written key is a
    // result candidate: with deletions or exclude masks the final top-k
    // filters the keys itself and does not read the bins, and the dense
    // scan's running bound must not count keys the filter would drop
    const bool count_keys = a.count_bins && a.dead == nullptr && a.qexclude == nullptr;

    // unit entry: {first row, chunk, first query slot, rows << 16 | queries};
    // lane s < queries holds query s's id and mask; for a single-query unit,
    // lane j also holds the query's j-th mask bit (from its slot, so that no
    // load waits for the query id)
    auto load_slots = [&](const int4& e, int& qid, uint64_t& m0, uint64_t& m1, uint32_t& sb) {
        qid = 0;
        m0 = 0;
        m1 = 0;
        sb = 0;
        const int qn = e.w & 0xFFFF;
        if (lane < qn) {
            qid = a.qlist[e.z + lane];
            const ulonglong2 m = reinterpret_cast<const ulonglong2*>(a.qmask_slot)[e.z + lane];
            m0 = m.x;
            m1 = m.y;
        }
        if (qn == 1) sb = a.slot_bits[int64_t(e.z) * kSlotBits + lane];
    };

    // Request a unit's planes into the buffer; returns the number of planes it
    // then holds, or -1 when the test must read global planes. A single-query
    // unit needs no union: its planes are the query's mask bits in increasing
    // order, which its slot carries (lane j holds bit j in sb).
    auto request_planes = [&](const int4& e, uint64_t m0, uint64_t m1, uint32_t sb) -> int {
        if ((e.w & 0xFFFF) == 1 && a.n_or == 0) {
            const uint64_t x = __shfl_sync(0xffffffffu, m0, 0), y = __shfl_sync(0xffffffffu, m1, 0);
            const int nb = __popcll(x) + (W > 1 ? __popcll(y) : 0);
            if (nb > kPlaneSlots) return -1;
            const uint32_t* src = a.planes + int64_t(e.y) * NPL * 16 + (lane & 3) * 4;
#pragma unroll
            for (int t = 0; t < kPlaneSlots / 8; ++t) {
                const int j = (lane >> 2) + 8 * t;
                const int bit = int(__shfl_sync(0xffffffffu, sb, j));
                if (j < nb) cp_async16_cg(pbuf + j * 16 + (lane & 3) * 4, src + bit * 16);
            }
            return nb;
        }
        uint64_t x = m0, y = m1;
        warp_or2(x, y);
        if (!issue_planes<W>(a, e.y, x, y, pbuf, s_tab, s_inv, lane)) return -1;
        return __popcll(x) + (W > 1 ? __popcll(y) : 0);
    };

    // query vectors of a unit -> shared memory by cp.async
    auto stage_queries = [&](int qn, int qid) {
        for (int i0 = 0; i0 < qn * np; i0 += 32) {
            const int idx = i0 + lane;
            const int sq = idx / np;
            const int qg = __shfl_sync(0xffffffffu, qid, sq < qn ? sq : qn - 1);
            if (idx < qn * np) cp_async16(s_q + idx, a.queries + int64_t(qg) * d + 16 * (idx - sq * np));
        }
    };

    // Test a unit whose planes are in the buffer (held >= 0) or in global
    // memory: pass words -> pass[s][blk]; returns the OR over queries in `any`
    // and, in lane s, query s's survivor count (general path only).
    auto test_unit = [&](const int4& e, int qid, uint64_t m0, uint64_t m1, int held, uint32_t* pass, uint32_t& any,
                         uint32_t& mycnt) {
        const int len = e.w >> 16;
        const int qn = e.w & 0xFFFF;
        const uint32_t valid = len >= 32 * (blk + 1) ? 0xFFFFFFFFu
                             : (len <= 32 * blk ? 0u : ((1u << (len - 32 * blk)) - 1u));
        any = 0;
        mycnt = 0;
        if (qn == 1 && held >= 0 && a.n_or == 0) {
            // the buffer holds exactly the query's planes, in bit order
            const int h0 = (held + 1) >> 1;
            const int j1 = half ? held : h0;
            int j = half ? h0 : 0;
            uint32_t acc = 0xFFFFFFFFu;
            for (; j + 4 <= j1; j += 4)
                acc &= pbuf[j * 16 + blk] & pbuf[(j + 1) * 16 + blk] & pbuf[(j + 2) * 16 + blk] &
                       pbuf[(j + 3) * 16 + blk];
            for (; j < j1; ++j) acc &= pbuf[j * 16 + blk];
            acc &= __shfl_xor_sync(0xffffffffu, acc, 16);
            any = acc & valid;
            return;
        }
        const uint32_t* gpl = a.planes + int64_t(e.y) * NPL * 16 + blk;
        // AND of the planes of bits[j0 .. j1) for this lane's 32-row block:
        // four independent bit -> slot -> plane chains per step
        auto and_bits = [&](const uint8_t* bits, int j0, int j1) -> uint32_t {
            uint32_t acc = 0xFFFFFFFFu;
            if (held >= 0) {
                int j = j0;
                for (; j + 4 <= j1; j += 4) {
                    const int b0 = __ldg(bits + j), b1 = __ldg(bits + j + 1);
                    const int b2 = __ldg(bits + j + 2), b3 = __ldg(bits + j + 3);
                    const int s0 = s_tab[b0], s1 = s_tab[b1], s2 = s_tab[b2], s3 = s_tab[b3];
                    acc &= pbuf[s0 * 16 + blk] & pbuf[s1 * 16 + blk] & pbuf[s2 * 16 + blk] & pbuf[s3 * 16 + blk];
                }
                for (; j < j1; ++j) acc &= pbuf[s_tab[__ldg(bits + j)] * 16 + blk];
            } else {
                for (int j = j0; j < j1; ++j) acc &= __ldg(gpl + __ldg(bits + j) * 16);
            }
            return acc;
        };
        for (int s = 0; s < qn; ++s) {
            const int qg = __shfl_sync(0xffffffffu, qid, s);
            uint32_t acc;
            if (a.n_or == 0) {
                // query s's mask bits: from its slot when the buffer holds the
                // planes (then it has at most kPlaneSlots <= kSlotBits of them),
                // else from the query's own list; the two half-warps take the
                // two halves of them
                const uint64_t x = __shfl_sync(0xffffffffu, m0, s), y = __shfl_sync(0xffffffffu, m1, s);
                const int nb = __popcll(x) + (W > 1 ? __popcll(y) : 0);
                const int h0 = (nb + 1) >> 1;
                const uint8_t* bits = held >= 0 ? a.slot_bits + int64_t(e.z + s) * kSlotBits
                                                : a.qbits + int64_t(qg) * kMaskBitsMax;
                acc = and_bits(bits, half ? h0 : 0, half ? nb : h0);
                acc &= __shfl_xor_sync(0xffffffffu, acc, 16);
            } else {
                // alternative masks: the OR over them of each one's AND (the
                // slot's mask, the union, chose the planes)
                const int n_alt = 1 + a.n_or;
                acc = 0;
                for (int alt = 0; alt < n_alt; ++alt) {
                    const int64_t row = int64_t(qg) * n_alt + alt;
                    const int nb = __ldg(a.qnbits + row);
                    const int h0 = (nb + 1) >> 1;
                    uint32_t ac = and_bits(a.qbits + row * kMaskBitsMax, half ? h0 : 0, half ? nb : h0);
                    ac &= __shfl_xor_sync(0xffffffffu, ac, 16);
                    acc |= ac;
                }
            }
            acc &= valid;
            if (half == 0) pass[s * 16 + blk] = acc;
            any |= acc;
            // survivors of query s: half 0 holds the 16 pass words; the full
            // 32-lane reduction leaves the total in every lane
            uint32_t c = half == 0 ? uint32_t(__popc(acc)) : 0u;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
            if (lane == s) mycnt = c;
        }
    };

    // After a unit's test: survivor row offsets -> sv, one reservation per
    // query (lane s, the reply lands in `base`), the first R survivors' rows
    // copied into `srow` (cp.async, in the group the caller commits next) and
    // the next ones prefetched into L2. Returns the number of survivors.
    auto settle_unit = [&](const int4& e, int qid, bool single, uint32_t any, uint32_t mycnt, uint16_t* sv,
                           int4* srow, uint32_t& base) -> int {
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
                sv[pos++] = uint16_t(32 * blk + i);
            }
        }
        if (single && lane == 0) mycnt = uint32_t(nsurv);
        base = 0;
        if (lane < (e.w & 0xFFFF) && mycnt) {
            base = atomicAdd(&a.cand_cnt[int64_t(qid) * kCntStride], mycnt);
            atomicAdd(&a.eligible_cnt[int64_t(qid) * (kCntStride / 2)], (unsigned long long)mycnt);
        }
        __syncwarp();
        if constexpr (R > 0) {
            constexpr int NPS = NP > 0 ? NP : 1;
            const int ns = nsurv < R ? nsurv : R;
            for (int c = lane; c < ns * NPS; c += 32) {
                const int idx = c / NPS, p = c - idx * NPS;
                cp_async16_cg(srow + c, a.items + (int64_t(e.x) + sv[idx]) * d + 16 * p);
            }
        }
        const int npf = nsurv < R + 64 ? nsurv : R + 64;
        for (int idx = R + lane; idx < npf; idx += 32) {
            const int8_t* row = a.items + (int64_t(e.x) + sv[idx]) * d;
            for (int o = 0; o < d; o += 32) prefetch_l2(row + o);
        }
        return nsurv;
    };

    // prologue: test unit 0; groups planes(0) [waited], planes(1), queries(0)
    int4 e_cur = a.units[u];
    int4 e_nxt = make_int4(0, 0, 0, 0), e_n2 = make_int4(0, 0, 0, 0);
    int u_n1 = draw(), u_n2 = draw();
    if (u_n1 < n_units) e_nxt = a.units[u_n1];
    if (u_n2 < n_units) e_n2 = a.units[u_n2];
    int qid_c, qid_n = 0;
    uint64_t m0_n = 0, m1_n = 0;
    uint32_t sb_n = 0;
    int held;          // planes the buffer holds for the next unit to test (-1: global)
    uint32_t base_c;   // lane s: reservation of query s of the unit being scored
    int nsurv_c;       // survivors of the unit being scored
    bool single_c;     // it took the single-query path
    {
        uint64_t m0_c, m1_c;
        uint32_t sb_c;
        load_slots(e_cur, qid_c, m0_c, m1_c, sb_c);
        if (u_n1 < n_units) load_slots(e_nxt, qid_n, m0_n, m1_n, sb_n);
        const int held0 = request_planes(e_cur, m0_c, m1_c, sb_c);
        cp_async_commit();
        cp_async_wait_group<0>();
        __syncwarp();
        uint32_t any, mycnt;
        test_unit(e_cur, qid_c, m0_c, m1_c, held0, pass2, any, mycnt);
        single_c = (e_cur.w & 0xFFFF) == 1 && held0 >= 0;
        __syncwarp();
        held = u_n1 < n_units ? request_planes(e_nxt, m0_n, m1_n, sb_n) : -1;
        cp_async_commit();
        nsurv_c = settle_unit(e_cur, qid_c, single_c, any, mycnt, surv2, srow2, base_c);
    }
    stage_queries(e_cur.w & 0xFFFF, qid_c);
    cp_async_commit();
    int cb = 0;

    while (u < n_units) {
        const int u_n3 = draw();
        const bool has_n1 = u_n1 < n_units;
        const bool has_n2 = u_n2 < n_units;
        const bool has_n3 = u_n3 < n_units;

        // background loads: the entry three units ahead, the slots of the unit
        // two ahead (whose entry arrived during the previous unit)
        int4 e_n3 = make_int4(0, 0, 0, 0);
        if (has_n3) e_n3 = a.units[u_n3];
        int qid_2 = 0;
        uint64_t m0_2 = 0, m1_2 = 0;
        uint32_t sb_2 = 0;
        if (has_n2) load_slots(e_n2, qid_2, m0_2, m1_2, sb_2);

        // test the next unit: its planes are the older of the (at most two)
        // pending groups [planes(u+1), queries(u)]
        int nsurv_n = 0;
        uint32_t base_n = 0;
        bool single_n = false;
        if (has_n1) {
            cp_async_wait_group<1>();
            __syncwarp();
            uint32_t any, mycnt;
            test_unit(e_nxt, qid_n, m0_n, m1_n, held, pass2 + (cb ^ 1) * kQMax * 16, any, mycnt);
            single_n = (e_nxt.w & 0xFFFF) == 1 && held >= 0;
            __syncwarp();
            held = has_n2 ? request_planes(e_n2, m0_2, m1_2, sb_2) : -1;
            cp_async_commit();
            nsurv_n = settle_unit(e_nxt, qid_n, single_n, any, mycnt, surv2 + (cb ^ 1) * kWarpItems,
                                  srow2 + (cb ^ 1) * R * NP, base_n);
        } else {
            cp_async_commit();  // two groups per unit, always
        }

        // score this unit: its query vectors are pending at most behind [planes(u+2)]
        cp_async_wait_group<1>();
        __syncwarp();
        const int64_t ib = e_cur.x;
        const int qn = e_cur.w & 0xFFFF;
        const uint16_t* surv = surv2 + cb * kWarpItems;
        const uint32_t* s_pass = pass2 + cb * kQMax * 16;
        const int4* srow = srow2 + cb * R * NP;  // the first R survivors' rows
        if (single_c) {
            // every survivor is a key of the one query, in survivor order
            const int qg = __shfl_sync(0xffffffffu, qid_c, 0);
            const uint32_t base0 = __shfl_sync(0xffffffffu, base_c, 0);
            uint64_t* cand = a.cand + int64_t(qg) * a.cap;
            const int2 sc = a.qscale[qg];
            uint32_t* qh = a.qhist + int64_t(qg) * kTcBins;
            for (int c0 = 0; c0 < nsurv_c; c0 += 32) {
                const int idx = c0 + lane;
                if (idx < nsurv_c) {
                    const int64_t i = ib + surv[idx];
                    const int4* rp = reinterpret_cast<const int4*>(a.items + i * d);
                    int32_t acc0 = 0, acc1 = 0;
                    if (NP > 0) {
                        int4 row[NP > 0 ? NP : 1];
                        if (idx < R) {
#pragma unroll
                            for (int p = 0; p < (NP > 0 ? NP : 1); ++p) row[p] = srow[idx * NP + p];
                        } else {
#pragma unroll
                            for (int p = 0; p < (NP > 0 ? NP : 1); ++p) row[p] = __ldg(rp + p);
                        }
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
                    if (count_keys) count_bin(qh, (score - sc.x) >> sc.y, __activemask());
                }
            }
        } else {
            // a key's slot is its ballot rank among this unit's survivors of
            // the same query
            uint32_t run = 0;  // lane s: keys of query s written so far
            for (int c0 = 0; c0 < nsurv_c; c0 += 32) {
                const int idx = c0 + lane;
                int off = -1;
                int64_t i = 0;
                int4 row[NP > 0 ? NP : 1];
                const int4* rp = nullptr;
                if (idx < nsurv_c) {
                    off = surv[idx];
                    i = ib + off;
                    rp = reinterpret_cast<const int4*>(a.items + i * d);
                    if (NP > 0) {
                        if (idx < R) {
#pragma unroll
                            for (int p = 0; p < (NP > 0 ? NP : 1); ++p) row[p] = srow[idx * NP + p];
                        } else {
#pragma unroll
                            for (int p = 0; p < (NP > 0 ? NP : 1); ++p) row[p] = __ldg(rp + p);
                        }
                    }
                }
                const uint32_t* pw = s_pass + (off >= 0 ? (off >> 5) : 0);
                const int bit = off & 31;
                for (int s = 0; s < qn; ++s) {
                    const bool on = off >= 0 && ((pw[s * 16] >> bit) & 1u);
                    const unsigned bal = __ballot_sync(0xffffffffu, on);
                    if (bal == 0u) continue;
                    const uint32_t slot0 = __shfl_sync(0xffffffffu, base_c, s) + __shfl_sync(0xffffffffu, run, s);
                    const int qg = __shfl_sync(0xffffffffu, qid_c, s);
                    if (on) {
                        const int2 sc = a.qscale[qg];
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
                        if (pos < uint64_t(a.cap)) a.cand[int64_t(qg) * a.cap + int64_t(pos)] = pack_key(score, uint32_t(i));
                        if (count_keys) count_bin(a.qhist + int64_t(qg) * kTcBins, (score - sc.x) >> sc.y, bal);
                    }
                    if (lane == s) run += __popc(bal);
                }
            }
        }

        // the next unit's query vectors (group queries(u+1))
        __syncwarp();
        if (has_n1) stage_queries(e_nxt.w & 0xFFFF, qid_n);
        cp_async_commit();

        e_cur = e_nxt;
        e_nxt = e_n2;
        e_n2 = e_n3;
        qid_c = qid_n;
        qid_n = qid_2;
        m0_n = m0_2;
        m1_n = m1_2;
        base_c = base_n;
        nsurv_c = nsurv_n;
        single_c = single_n;
        cb ^= 1;
        u = u_n1;
        u_n1 = u_n2;
        u_n2 = u_n3;
    }
    cp_async_wait_all();  // no copy may land after the warp has left
}

template <int NP, int W>
static cudaError_t launch_variant(const SearchArgs& a, int num_sms, cudaStream_t s)
{
    const size_t smem = scan_smem_bytes(a.d, W);
    const void* fn = reinterpret_cast<const void*>(scan_kernel<NP, W>);
    const int slot = 1 + (NP == 4 ? 0 : NP == 8 ? 1 : 2) + 3 * (W - 1);
    cudaError_t e = ensure_smem_attr(fn, int(scan_smem_bytes(ST_MAX_D, W)));
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
    return launch_dep(scan_kernel<NP, W>, dim3(num_sms * occ), dim3(kScanBlock), smem, s, a);
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
