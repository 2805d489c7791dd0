// Dense-unit list scan on the 5th-generation tensor cores.
//
// Same method as the warp scan (scan.cu): inside every probed list, the Bloom
// test (sig & mask) == mask decides eligibility, only eligible items are
// scored by the int8 inner product, and the scores feed the final top-k
// (SilverTorch: Index as Model, section on redesigning each stage as a pure
// PyTorch module, Bloom index filter and fused Int8 ANN paragraphs). When many
// queries probe the same list, a unit (512 rows x up to 32 of those queries)
// is a dense int8 contraction, and it runs here as tensor-core tiles instead
// of per-pair dp4a.
//
// A persistent CTA per SM, warp-specialized, its roles handing units on
// through mbarriers so that several units are in flight at once:
//   * two producer warps, on different SM sub-partitions, taking alternate
//     units: the unit's query slots (three of the warp's units ahead), its
//     signature bit-planes (the union of its queries' mask bits, by cp.async,
//     two of its units ahead, into the unit's slot of the unit ring, where they
//     stay until its epilogue is done), then its rows, as whole 128-row TMA
//     tiles in the canonical 128-byte (d = 128) or 64-byte (d = 64) swizzled
//     K-major layout of an operand stage, and the unit's query vectors. The
//     lists here have many queries or many eligible rows, so nearly every row
//     block holds a survivor of some query: testing first to skip row blocks
//     cost the producers more than the reads it saved;
//   * MMA warp: one thread issues tcgen05.mma kind::i8 (M = 128 rows, N = the
//     unit's queries rounded up to 16, K = 32) into int32 accumulators in TMEM
//     and commits to mbarriers that free the operand stage and hand the
//     accumulators to an epilogue;
//   * four epilogue warpgroups, one per TMEM accumulator stage (every fourth
//     unit each): lane q of each warp runs the Bloom test of query q on the
//     warp's four 32-row blocks (the AND of the unit's planes of its mask
//     bits); each thread reads its row's scores (tcgen05.ld) and keeps a key
//     only if the row passes the query's test and its score reaches the
//     query's running bound (below), as one bit per query; a 32 x 32 bit
//     transpose across the warp turns the pass words into these per-row words
//     and the kept words into per-query row masks, whose popcounts are the
//     warp's key counts. Each warp reserves its slots with one atomic per query
//     (all in flight at once) and writes its keys at the query's base plus the
//     key's rank in the row mask, counting each in its score bin with one
//     atomic (the keys of one query in one 32-row block rarely share a bin, so
//     grouping them first costs more than it saves).
//
// Running top-k bound. Intermediate results should stay on chip (Andromeda
// review, section on why the bottleneck moved from compute to bandwidth), so
// keys that can no longer enter a query's top-k are not written at all. Every
// written key is a real candidate, so if at least k written keys have scores
// >= T, the query's k-th best score is >= T and any key below T can be
// dropped. Every written key is counted in the query's 1024
// bins over its possible score range [-S, S], S = 128 sum_j |q_j| (bin b
// holds scores in [-S + b 2^sh, -S + (b+1) 2^sh)); when a unit wrote at least
// max(kTcBoundMinKeys, k / 8) keys of a query, the bins from its bound upward give
// the highest bin edge with k written keys at or above it, published with
// atomicMax. The bound only grows and the final top-k is unchanged (exact).
// With deletions or exclude masks this scan applies the post-filter before it
// counts a key, and the warp scan (which writes its keys unfiltered for the
// final top-k to filter) counts none, so every counted key is a candidate.
//
// Waits are bounded: a wait that runs out sets an error bit and an abort flag;
// every role then leaves its loop (its own waits are bounded too), and the CTA
// frees its TMEM after a last bounded wait for its copies and MMAs in flight.
#include "tc_ptx.cuh"

namespace st {

constexpr int kTcRows = kWarpItems;      // rows per unit
constexpr int kTcPlaneSlots = 24;        // planes a unit's ring slot holds (a wider union reads global planes)
constexpr uint32_t kTcWaitLimit = 1u << 22;
// Units whose data are held at once. A producer refills the slot of unit
// j - 8 (with unit j + 4) only after the MMAs of unit j - S (operand stages
// S = 2 or 4) are done; those of unit j - 4 then are too, and they waited for
// the epilogue of unit j - 8 (epilogue groups 4) to free its accumulators.
constexpr int kTcMeta = 12;
constexpr uint32_t kTcBoundMinKeys = 16; // least keys of a query in one unit that make it re-read its bound (else k / 8)
constexpr int kTcEpiGroups = 4;         // epilogue warpgroups, one per TMEM accumulator stage
constexpr int kTcProducers = 2;         // producer warps (units alternate between them)
constexpr int kTcProd1Warp = 2 + 4 * kTcEpiGroups;  // the second producer: the last warp
constexpr int kTcThreads = 32 * (2 + 4 * kTcEpiGroups + 1);
static_assert(kTcProducers == 2, "warp 0 and the last warp produce");
constexpr int kTcAccCols = 4 * kTcQMax;  // TMEM columns of one unit's accumulators (4 row blocks)
constexpr int kTcTmemCols = kTcEpiGroups * kTcAccCols;

// operand stages (rows and queries of one unit each)
template <int D>
__host__ __device__ constexpr int tc_stages()
{
    return D == 64 ? 4 : 2;
}

struct TcMeta {                          // one unit, from its slots to its epilogue
    int4 e;                              // {first row, plane block, first slot, rows << 16 | queries}
    uint32_t planes[kTcPlaneSlots][16];  // the signature bit-planes of the union of its queries' masks
    int32_t qid[kTcQMax];
    unsigned long long qm[kTcQMax][2];   // the queries' masks
    uint32_t thr[kTcQMax];               // the queries' running bounds when the unit was loaded
    int32_t qbase[kTcQMax], qsh[kTcQMax];  // score bins: lowest possible score, bin shift
    uint8_t tab[kMaskBitsMax];           // signature bit -> plane slot
    uint8_t inv[kTcPlaneSlots];          // plane slot -> signature bit
    int32_t held;                        // planes in the buffer (-1: the test reads global planes)
    uint32_t mbmask;                     // 128-row blocks holding rows of the unit (MMAs issued for them)
};

struct TcEpi {                           // one epilogue warpgroup's per-query key counts (two units)
    uint32_t cnt[2][kTcQMax];
    uint32_t wbase[4][kTcQMax];          // per warp: query q's next key slot in the current row block
    uint32_t wcol[4][kTcQMax];           // per warp: query q's kept rows of the current row block
};

// 32 x 32 bit-matrix transpose across a warp: lane i holds row i (bit j =
// element (i, j)) and gets column i (bit j = element (j, i)), by exchanging
// ever smaller blocks between lanes
__device__ __forceinline__ uint32_t warp_transpose32(uint32_t x, int lane)
{
    const uint32_t lo[5] = {0x0000FFFFu, 0x00FF00FFu, 0x0F0F0F0Fu, 0x33333333u, 0x55555555u};
#pragma unroll
    for (int i = 0; i < 5; ++i) {
        const int sft = 16 >> i;
        const uint32_t y = __shfl_xor_sync(0xffffffffu, x, sft);
        x = (lane & sft) ? ((x & ~lo[i]) | ((y & ~lo[i]) >> sft)) : ((x & lo[i]) | ((y & lo[i]) << sft));
    }
    return x;
}

#ifdef ST_TC_PROF
// Per-CTA cycle counters of the pipeline roles (a measuring build only).
static __device__ unsigned long long g_tc_prof[1024][16];
#define TC_T0(v) const long long v = clock64()
#define TC_ACC(slot, v) atomicAdd(&g_tc_prof[blockIdx.x][slot], (unsigned long long)(clock64() - (v)))
#else
#define TC_T0(v)
#define TC_ACC(slot, v)
#endif

template <int D>
__device__ __forceinline__ uint32_t swz(int r, int c)
{
    // canonical swizzled K-major layout: 8-row atoms of 8 * D bytes; the
    // 16-byte chunk c of row r is XORed with the row's place in the atom
    const int x = D == 128 ? (r & 7) : ((r & 7) >> 1);
    return uint32_t((r >> 3) * (8 * D) + (r & 7) * D + ((c ^ x) << 4));
}

// Dynamic shared memory of one CTA, in order: operand stages (rows, then
// query vectors), two plane buffers, the unit ring, the epilogue counts. The
// kernel carves its buffers from these offsets and the launch requests
// tc_dyn_smem() (the end plus the slack for aligning the base to 1024 bytes,
// which the swizzled operand layouts need).
template <int D>
struct TcLayout {
    static constexpr size_t kA = 0;
    static constexpr size_t kB = kA + size_t(tc_stages<D>()) * kTcRows * D;
    static constexpr size_t kMeta = kB + size_t(tc_stages<D>()) * kTcQMax * D;
    static constexpr size_t kEpi = kMeta + size_t(kTcMeta) * sizeof(TcMeta);
    static constexpr size_t kEnd = kEpi + size_t(kTcEpiGroups) * sizeof(TcEpi);
    static_assert(kMeta % alignof(TcMeta) == 0 && kEpi % alignof(TcEpi) == 0, "aligned carve-up");
};

template <int D>
__host__ __device__ constexpr size_t tc_dyn_smem()
{
    return TcLayout<D>::kEnd + 1024;
}

template <int D, int W>
__global__ void __launch_bounds__(kTcThreads, 1)
scan_tc_kernel(SearchArgs a, const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap tmap128)
{
    dep_enter();
    const int n_units = a.ctl->n_dense < a.max_units ? a.ctl->n_dense : a.max_units;
    if (int(blockIdx.x) >= n_units) return;  // CTA-uniform, before any allocation

    constexpr int S = tc_stages<D>();
    constexpr int NPL = 64 * W;          // planes per chunk
    constexpr int CH = D / 16;           // 16-byte chunks per row
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[S], empty_bar[S], acc_full[kTcEpiGroups], acc_empty[kTcEpiGroups],
        meta_full[kTcMeta];
    __shared__ uint32_t s_tmem;
    __shared__ volatile int s_abort;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t raw_sa = smem_u32(smem_raw);
    unsigned char* const base = smem_raw + (((raw_sa + 1023u) & ~1023u) - raw_sa);
    using L = TcLayout<D>;
    unsigned char* const Abuf = base + L::kA;                                 // [S][kTcRows * D]
    unsigned char* const Bbuf = base + L::kB;                                 // [S][kTcQMax * D]
    TcMeta* const meta = reinterpret_cast<TcMeta*>(base + L::kMeta);          // [kTcMeta]
    TcEpi* const epi = reinterpret_cast<TcEpi*>(base + L::kEpi);              // [kTcEpiGroups]

    if (tid == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full_bar[i], 2);   // the TMA byte count's arrival + the query vectors' arrival
            mbar_init(&empty_bar[i], 1);  // the MMAs reading the stage are done
        }
        for (int i = 0; i < kTcEpiGroups; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 1);
        }
        for (int i = 0; i < kTcMeta; ++i) mbar_init(&meta_full[i], 1);  // the unit's data are complete
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(&s_tmem, kTcTmemCols);
        tmem_relinquish();
    }
    for (int i = tid; i < kTcEpiGroups * 2 * kTcQMax; i += kTcThreads)
        epi[i / (2 * kTcQMax)].cnt[(i / kTcQMax) & 1][i % kTcQMax] = 0;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    const int n_iter = (n_units - int(blockIdx.x) + int(gridDim.x) - 1) / int(gridDim.x);
    auto unit_entry = [&](int j) { return a.units_tc[blockIdx.x + int64_t(j) * gridDim.x]; };
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
        if (s_abort) return false;
        if (mbar_wait(bar, parity, kTcWaitLimit)) return true;
        s_abort = 1;
        set_error(a.err, kErrTcWait);
        return false;
    };

    if (warp == 0 || warp == kTcProd1Warp) {
        // ============================== producers =============================
        // producer `pid` takes units pid, pid + 2, pid + 4, ... with plane
        // buffers 2 pid and 2 pid + 1 (alternate units of its own)
        const int pid = warp == 0 ? 0 : 1;
        constexpr int P2 = kTcProducers;
        struct Slots {
            int4 e;
            int qid;
            unsigned long long m0, m1;
            uint32_t thr;
            int2 sc;
        };
        auto load_slots = [&](int j) {
            Slots r;
            r.e = unit_entry(j);
            r.qid = 0;
            r.m0 = r.m1 = 0;
            r.thr = 0;
            r.sc = make_int2(0, 0);
            if (lane < (r.e.w & 0xFFFF)) {
                r.qid = a.qlist[r.e.z + lane];
                const ulonglong2 mk = reinterpret_cast<const ulonglong2*>(a.qmask_slot)[r.e.z + lane];
                r.m0 = mk.x;
                r.m1 = mk.y;
            }
            return r;
        };
        // a second round of loads that depend on the query ids
        auto finish_slots = [&](Slots& r) {
            if (lane < (r.e.w & 0xFFFF)) {
                r.thr = __ldcg(a.score_rng + int64_t(r.qid) * kCntStride + kRngThr);
                r.sc = a.qscale[r.qid];
            }
        };
        // slots -> meta[m]; the union's planes -> meta[m].planes
        auto store_and_request = [&](int m, const Slots& r) {
            const int qn = r.e.w & 0xFFFF;
            TcMeta& mt = meta[m];
            if (lane == 0) mt.e = r.e;
            if (lane < qn) {
                mt.qid[lane] = r.qid;
                mt.qm[lane][0] = r.m0;
                mt.qm[lane][1] = r.m1;
                mt.thr[lane] = r.thr;
                mt.qbase[lane] = r.sc.x;
                mt.qsh[lane] = r.sc.y;
            }
            unsigned long long u0 = r.m0, u1 = r.m1;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                u0 |= __shfl_xor_sync(0xffffffffu, u0, off);
                u1 |= __shfl_xor_sync(0xffffffffu, u1, off);
            }
            if (W == 1) u1 = 0;
            const int n0 = __popcll(u0);
            const int nb = n0 + __popcll(u1);
            if (lane == 0) mt.held = nb > kTcPlaneSlots ? -1 : nb;
            if (nb > kTcPlaneSlots) {
                __syncwarp();
                return;
            }
#pragma unroll
            for (int rr = 0; rr < 2 * W; ++rr) {
                const int b = lane + 32 * rr;
                const unsigned long long word = b < 64 ? u0 : u1;
                const unsigned long long below = (b & 63) ? (word & ((1ull << (b & 63)) - 1ull)) : 0ull;
                const int slot = (b < 64 ? 0 : n0) + __popcll(below);
                const bool on = (word >> (b & 63)) & 1ull;
                mt.tab[b] = on ? uint8_t(slot) : uint8_t(0);
                if (on) mt.inv[slot] = uint8_t(b);
            }
            __syncwarp();
            uint32_t* dst = &mt.planes[0][0];
            const uint32_t* src = a.planes + int64_t(r.e.y) * NPL * 16;
            for (int item = lane; item < 4 * nb; item += 32)
                cp_async16_cg(dst + item * 4, src + mt.inv[item >> 2] * 16 + (item & 3) * 4);
        };
        // rows and query vectors of meta[m] -> operand stage s
        auto issue_rows = [&](int m, int s) {
            TcMeta& mt = meta[m];
            const int4 e = mt.e;
            const int qn = e.w & 0xFFFF;
            unsigned char* A = Abuf + s * kTcRows * D;
            unsigned char* Bq = Bbuf + s * kTcQMax * D;
            // every 128-row tile holding rows of the unit, by TMA (rows past
            // the end of the index read as zeros; rows past the unit's pass
            // no Bloom test in the epilogue)
            const int nblk = ((e.w >> 16) + 127) >> 7;
            const uint32_t mb = nblk > 0 ? (1u << nblk) - 1u : 0u;
            if (lane == 0) {
                mt.mbmask = mb;
                mbar_arrive_expect_tx(&full_bar[s], uint32_t(nblk) * 128u * D);
                for (int r4 = 0; r4 < nblk; ++r4) tma_load_2d(A + r4 * 128 * D, &tmap128, 0, e.x + 128 * r4, &full_bar[s]);
            }
            for (int item = lane; item < qn * CH; item += 32) {
                const int q = item / CH, c = item - q * CH;
                cp_async16(Bq + swz<D>(q, c), a.queries + int64_t(mt.qid[q]) * D + 16 * c);
            }
        };
        // the query vectors (cp.async) of the unit using stage s have landed:
        // make them visible to the tensor cores and count the stage's second
        // arrival
        auto gathers_done = [&](int s) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&full_bar[s]);
        };

        // prologue: slots and planes of this producer's first two units, slots
        // of its third in registers
        if (pid < n_iter) {
            Slots r0 = load_slots(pid);
            finish_slots(r0);
            store_and_request(pid % kTcMeta, r0);
        }
        cp_async_commit();
        if (pid + P2 < n_iter) {
            Slots r1 = load_slots(pid + P2);
            finish_slots(r1);
            store_and_request((pid + P2) % kTcMeta, r1);
        }
        cp_async_commit();
        cp_async_commit();
        Slots nxt;
        if (pid + 2 * P2 < n_iter) {
            nxt = load_slots(pid + 2 * P2);
            finish_slots(nxt);
        }
        int last = -1;  // this producer's latest unit
        for (int j = pid; j < n_iter; j += P2) {
            const int s = j % S, m = j % kTcMeta;
            TC_T0(t0);
            // the queries' current bounds (they only grow; the ones loaded with
            // the slots are several units old), stored before the epilogue gets
            // the unit, so both of its passes see one value per query
            uint32_t thr_now = 0;
            const int qn_j = meta[m].e.w & 0xFFFF;
            if (lane < qn_j) thr_now = __ldcg(a.score_rng + int64_t(meta[m].qid[lane]) * kCntStride + kRngThr);
            // unit j's planes (its epilogue reads them) and the previous unit's rows
            cp_async_wait_group<1>();
            __syncwarp();
            if (last >= 0) gathers_done(last % S);
            TC_T0(t1);
            TC_T0(t2);
            TC_T0(t3);
            if (j >= S && !wait(&empty_bar[s], uint32_t(j / S - 1) & 1u)) break;
            TC_T0(t4);
            issue_rows(m, s);
            cp_async_commit();
            if (lane < qn_j && thr_now > meta[m].thr[lane]) meta[m].thr[lane] = thr_now;
            __syncwarp();
            if (lane == 0) mbar_arrive(&meta_full[m]);  // slots, planes, bounds and row blocks of unit j
            last = j;
            TC_T0(t5);
            if (j + 2 * P2 < n_iter) store_and_request((j + 2 * P2) % kTcMeta, nxt);
            cp_async_commit();
            TC_T0(t6);
            if (j + 3 * P2 < n_iter) {
                nxt = load_slots(j + 3 * P2);
                finish_slots(nxt);
            }
            if (lane == 0) {
                TC_ACC(1, t0); TC_ACC(2, t1); TC_ACC(3, t2); TC_ACC(4, t3); TC_ACC(5, t4); TC_ACC(6, t5); TC_ACC(7, t6);
            }
        }
        cp_async_wait_all();
        if (!s_abort && last >= 0) gathers_done(last % S);
    } else if (warp == 1) {
        // ================================ MMA =================================
        for (int j = 0; j < n_iter; ++j) {
            const int s = j % S, g = j % kTcEpiGroups, m = j % kTcMeta;
            TC_T0(t0);
            if (!wait(&full_bar[s], uint32_t(j / S) & 1u)) break;
            TC_T0(t1);
            if (j >= kTcEpiGroups && !wait(&acc_empty[g], uint32_t(j / kTcEpiGroups - 1) & 1u)) break;
            if (lane == 0) { TC_ACC(8, t0); TC_ACC(9, t1); }
            tc_fence_after();
            if (lane == 0) {
                const uint32_t mbm = meta[m].mbmask;
                if (mbm) {
                    const int qn = meta[m].e.w & 0xFFFF;
                    const uint32_t idesc = idesc_i8(128, (qn + 15) & ~15);
                    const uint32_t a0 = smem_u32(Abuf + s * kTcRows * D), b0 = smem_u32(Bbuf + s * kTcQMax * D);
                    for (int mb = 0; mb < 4; ++mb) {
                        if (!((mbm >> mb) & 1u)) continue;
#pragma unroll
                        for (int ks = 0; ks < D / 32; ++ks)
                            tc_mma_i8(tmem + uint32_t(g * kTcAccCols + mb * kTcQMax),
                                      smem_desc_kmajor(a0 + mb * 128 * D + ks * 32, D),
                                      smem_desc_kmajor(b0 + ks * 32, D), idesc, ks > 0 ? 1u : 0u);
                    }
                    tc_commit(&acc_full[g]);
                    tc_commit(&empty_bar[s]);
                } else {
                    mbar_arrive(&acc_full[g]);
                    mbar_arrive(&empty_bar[s]);
                }
            }
            __syncwarp();
        }
    } else {
        // ============================== epilogue ==============================
        const int g = (warp - 2) >> 2;             // warpgroup: TMEM stage g, units j = g, g + G, ...
        const int gt = tid - 64 - 128 * g;         // thread within the warpgroup
        const int wq = warp & 3;                   // TMEM lane quarter of this warp
        TcEpi& E = epi[g];
        const bool filt = a.dead != nullptr || a.qexclude != nullptr;
        const uint32_t acc_base = tmem + (uint32_t(wq * 32) << 16) + uint32_t(g * kTcAccCols);
        // keys a query must gain in one unit before its bound is re-read
        const uint32_t bound_min = uint32_t(a.k / 8) > kTcBoundMinKeys ? uint32_t(a.k / 8) : kTcBoundMinKeys;
        for (int j = g, it = 0; j < n_iter; j += kTcEpiGroups, ++it) {
            const int m = j % kTcMeta;
            uint32_t* cnt = E.cnt[it & 1];
            TC_T0(e0);
            if (!wait(&meta_full[m], uint32_t(j / kTcMeta) & 1u)) break;
            if (!wait(&acc_full[g], uint32_t(j / kTcEpiGroups) & 1u)) break;
            if (gt == 0) TC_ACC(10 + (g & 1), e0);
            TC_T0(e1);
            tc_fence_after();
            const TcMeta& mt = meta[m];
            const uint32_t mbm = mt.mbmask;
            const int4 e = mt.e;
            const int qn = e.w & 0xFFFF;
            int bq_id = 0, bq_base = 0, bq_sh = 0;  // this lane's query for the bound update
            uint32_t bq_thr = 0;
            bool bq_go = false;
            if (mbm) {
                const int nsl = (qn + 15) >> 4;
                // the Bloom test of this warp's four 32-row blocks (4 mb + wq)
                // for query `lane`: the AND over its mask's bits of the unit's
                // planes (for alternative masks, the OR over them of each one's
                // AND), limited to the unit's rows
                uint32_t pw0 = 0, pw1 = 0, pw2 = 0, pw3 = 0;
                if (lane < qn) {
                    const int len = e.w >> 16, held = mt.held;
                    const uint32_t* gpl = a.planes + int64_t(e.y) * NPL * 16;
                    auto plane_word = [&](int b, int wb) -> uint32_t {
                        return held >= 0 ? mt.planes[mt.tab[b]][wb] : __ldg(gpl + b * 16 + wb);
                    };
                    auto and_mask = [&](uint64_t m0, uint64_t m1, uint32_t& v0, uint32_t& v1, uint32_t& v2, uint32_t& v3) {
                        v0 = v1 = v2 = v3 = 0xFFFFFFFFu;
                        for (int word = 0; word < W; ++word) {
                            unsigned long long mk = word == 0 ? m0 : m1;
                            while (mk) {
                                const int b = 64 * word + __ffsll(static_cast<long long>(mk)) - 1;
                                mk &= mk - 1;
                                v0 &= plane_word(b, wq);
                                v1 &= plane_word(b, 4 + wq);
                                v2 &= plane_word(b, 8 + wq);
                                v3 &= plane_word(b, 12 + wq);
                            }
                        }
                    };
                    if (a.n_or == 0) {
                        and_mask(mt.qm[lane][0], mt.qm[lane][1], pw0, pw1, pw2, pw3);
                    } else {
                        const int qid = mt.qid[lane];
                        for (int alt = 0; alt <= a.n_or; ++alt) {
                            const uint64_t* mk = alt == 0 ? a.qmasks + int64_t(qid) * W
                                                          : a.or_masks + (int64_t(qid) * a.n_or + alt - 1) * W;
                            uint32_t v0, v1, v2, v3;
                            and_mask(__ldg(mk), W > 1 ? __ldg(mk + 1) : 0ull, v0, v1, v2, v3);
                            pw0 |= v0;
                            pw1 |= v1;
                            pw2 |= v2;
                            pw3 |= v3;
                        }
                    }
                    auto rows_of = [&](int wb) -> uint32_t {
                        const int r0 = 32 * wb;
                        return len >= r0 + 32 ? 0xFFFFFFFFu : (len <= r0 ? 0u : ((1u << (len - r0)) - 1u));
                    };
                    pw0 &= rows_of(wq);
                    pw1 &= rows_of(4 + wq);
                    pw2 &= rows_of(8 + wq);
                    pw3 &= rows_of(12 + wq);
                    const uint32_t ne = __popc(pw0) + __popc(pw1) + __popc(pw2) + __popc(pw3);
                    if (ne) atomicAdd(&a.eligible_cnt[int64_t(mt.qid[lane]) * (kCntStride / 2)], (unsigned long long)ne);
                }
                // pass 1: this thread's kept pairs of each row block as a word
                // over the queries (bit q: the row passes query q's Bloom test
                // and its score reaches q's bound), and, transposed, lane q's
                // kept rows of query q
                uint32_t myc = 0;
                uint32_t kw[4] = {0u, 0u, 0u, 0u}, cw[4] = {0u, 0u, 0u, 0u};
#pragma unroll 1
                for (int mb = 0; mb < 4; ++mb) {
                    if (!((mbm >> mb) & 1u)) continue;  // warp-uniform
                    const int r = mb * 128 + wq * 32 + lane;
                    const uint32_t T = warp_transpose32(mb == 0 ? pw0 : mb == 1 ? pw1 : mb == 2 ? pw2 : pw3, lane);
                    uint32_t K = 0;
                    for (int sl = 0; sl < nsl; ++sl) {
                        uint32_t v[16];
                        tmem_ld16(acc_base + uint32_t(mb * kTcQMax + sl * 16), v);
                        tmem_wait_ld();
                        uint32_t k16 = 0;
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj)
                            if (int32_t(v[jj]) >= int32_t(mt.thr[sl * 16 + jj] ^ 0x80000000u)) k16 |= 1u << jj;
                        K |= k16 << (16 * sl);
                    }
                    K &= T;
                    if (filt) {
                        for (uint32_t kk = K; kk; kk &= kk - 1) {
                            const int q = __ffs(int(kk)) - 1;
                            if (!keep_item(a, mt.qid[q], int64_t(e.x) + r)) K &= ~(1u << q);
                        }
                    }
                    const uint32_t C = warp_transpose32(K, lane);
                    myc += __popc(C);
                    kw[0] = mb == 0 ? K : kw[0];
                    kw[1] = mb == 1 ? K : kw[1];
                    kw[2] = mb == 2 ? K : kw[2];
                    kw[3] = mb == 3 ? K : kw[3];
                    cw[0] = mb == 0 ? C : cw[0];
                    cw[1] = mb == 1 ? C : cw[1];
                    cw[2] = mb == 2 ? C : cw[2];
                    cw[3] = mb == 3 ? C : cw[3];
                }
                // this warp's slots: one atomic per query, all in flight at once
                uint32_t run = 0;
                if (lane < qn && myc) {
                    run = atomicAdd(&a.cand_cnt[int64_t(mt.qid[lane]) * kCntStride], myc);
                    atomicAdd(&cnt[lane], myc);
                }
                // pass 2: write the kept keys; a key's slot is its query's
                // base for the row block plus its rank among the block's kept
                // rows of that query (both from lane q, through shared memory)
                uint32_t* const wbase = E.wbase[wq];
                uint32_t* const wcol = E.wcol[wq];
#pragma unroll 1
                for (int mb = 0; mb < 4; ++mb) {
                    const uint32_t K = mb == 0 ? kw[0] : mb == 1 ? kw[1] : mb == 2 ? kw[2] : kw[3];
                    const uint32_t C = mb == 0 ? cw[0] : mb == 1 ? cw[1] : mb == 2 ? cw[2] : cw[3];
                    if (!__any_sync(0xffffffffu, K != 0u)) continue;  // then every C is 0 too
                    __syncwarp();
                    wbase[lane] = run;
                    wcol[lane] = C;
                    run += __popc(C);
                    __syncwarp();
                    const int r = mb * 128 + wq * 32 + lane;
                    const uint32_t id = uint32_t(e.x + r);
                    const uint32_t lt = lanemask_lt();
                    for (int sl = 0; sl < nsl; ++sl) {
                        uint32_t v[16];
                        tmem_ld16(acc_base + uint32_t(mb * kTcQMax + sl * 16), v);
                        tmem_wait_ld();
                        const uint32_t k16 = K >> (16 * sl);
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj) {
                            if (!((k16 >> jj) & 1u)) continue;
                            const int q = sl * 16 + jj;
                            const int32_t score = int32_t(v[jj]);
                            const uint32_t pos = wbase[q] + __popc(wcol[q] & lt);
                            const int qid = mt.qid[q];
                            if (int64_t(pos) < a.cap) a.cand[int64_t(qid) * a.cap + pos] = pack_key(score, id);
                            atomicAdd(a.qhist + int64_t(qid) * kTcBins + ((score - mt.qbase[q]) >> mt.qsh[q]), 1u);
                        }
                    }
                }
                named_barrier(1 + g, 128);  // the unit's key counts are complete
                // the bound update's inputs (below), read before the unit's
                // TMEM stage and ring slot are released: lane i takes query
                // wq + 4 i
                const int q = wq + 4 * lane;
                if (lane < kTcQMax / 4 && q < qn && cnt[q] >= bound_min) {
                    bq_go = true;
                    bq_id = mt.qid[q];
                    bq_thr = mt.thr[q];
                    bq_base = mt.qbase[q];
                    bq_sh = mt.qsh[q];
                }
            }
            if (gt < kTcQMax) E.cnt[(it + 1) & 1][gt] = 0;  // the counts of this group's next unit
            tc_fence_before();
            named_barrier(1 + g, 128);  // every read of TMEM and of meta[m] is done
            if (gt == 0) mbar_arrive(&acc_empty[g]);
            // then raise the bound of each query that gained at least
            // bound_min keys in the unit: the highest bin edge with at least k
            // written keys at or above it, from the query's bins at or above
            // its bound's bin (lane l reads bins 32 l .. 32 l + 31)
            constexpr int kPer = kTcBins / 32;
            for (unsigned go = __ballot_sync(0xffffffffu, bq_go); go; go &= go - 1) {
                const int i = __ffs(int(go)) - 1;
                const int qid = __shfl_sync(0xffffffffu, bq_id, i);
                const uint32_t thr = __shfl_sync(0xffffffffu, bq_thr, i);
                const int32_t qbase = __shfl_sync(0xffffffffu, bq_base, i);
                const int qsh = __shfl_sync(0xffffffffu, bq_sh, i);
                const uint4* gh = reinterpret_cast<const uint4*>(a.qhist + int64_t(qid) * kTcBins) + lane * (kPer / 4);
                const int tb = thr ? ((int32_t(thr ^ 0x80000000u) - qbase) >> qsh) : 0;
                uint32_t gv[kPer], tot = 0;
                const bool mine = kPer * lane + kPer - 1 >= tb;
#pragma unroll
                for (int r = 0; r < kPer / 4; ++r) {
                    const uint4 x = mine ? __ldcg(gh + r) : make_uint4(0, 0, 0, 0);
                    gv[4 * r] = x.x;
                    gv[4 * r + 1] = x.y;
                    gv[4 * r + 2] = x.z;
                    gv[4 * r + 3] = x.w;
                }
#pragma unroll
                for (int r = 0; r < kPer; ++r) tot += gv[r];
                uint32_t incl = tot;  // suffix sum over lanes >= this one
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const uint32_t o = __shfl_down_sync(0xffffffffu, incl, off);
                    if (lane + off < 32) incl += o;
                }
                uint32_t run = incl - tot, best = 0;  // keys in bins above this lane's
#pragma unroll
                for (int r = kPer - 1; r >= 0; --r) {
                    run += gv[r];
                    if (best == 0 && run >= uint32_t(a.k)) best = uint32_t(kPer * lane + r);
                }
                best = __reduce_max_sync(0xffffffffu, best);
                if (lane == 0 && best > 0) {
                    const int32_t T = qbase + int32_t(best << qsh);
                    atomicMax(a.score_rng + int64_t(qid) * kCntStride + kRngThr, uint32_t(T) ^ 0x80000000u);
                }
            }
            if (gt == 0) TC_ACC(12 + (g & 1), e1);
        }
    }

    // teardown: nothing of this CTA may be in flight when its TMEM is freed
#ifdef ST_TC_PROF
    if (tid == 0) g_tc_prof[blockIdx.x][0] += (unsigned long long)n_iter;
#endif
    __syncthreads();
    if (s_abort && tid == 0) {
        for (int i = 0; i < S; ++i) mbar_wait(&full_bar[i], 0, 1u << 12);
        for (int i = 0; i < kTcEpiGroups; ++i) mbar_wait(&acc_full[i], 0, 1u << 12);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, kTcTmemCols);
}

bool scan_tc_supported(int d) { return d == 64 || d == 128; }

#ifdef ST_TC_PROF
}  // namespace st
extern "C" int st_tc_prof_read(unsigned long long* host, int clear)
{
    cudaError_t e = cudaMemcpyFromSymbol(host, st::g_tc_prof, sizeof(st::g_tc_prof));
    if (e == cudaSuccess && clear) {
        static unsigned long long zero[1024][16];
        e = cudaMemcpyToSymbol(st::g_tc_prof, zero, sizeof(zero));
    }
    return int(e);
}
namespace st {
#endif

template <int D, int W>
static cudaError_t launch_tc(const SearchArgs& a, const void* tmaps, int num_sms, cudaStream_t s)
{
    const size_t smem = tc_dyn_smem<D>();
    const void* fn = reinterpret_cast<const void*>(scan_tc_kernel<D, W>);
    cudaError_t e = ensure_smem_attr(fn, int(smem));
    if (e != cudaSuccess) return e;
    CUtensorMap map32, map128;
    memcpy(&map32, tmaps, sizeof(CUtensorMap));
    memcpy(&map128, static_cast<const CUtensorMap*>(tmaps) + 1, sizeof(CUtensorMap));
    return launch_dep(scan_tc_kernel<D, W>, dim3(num_sms), dim3(kTcThreads), smem, s, a, map32, map128);
}

cudaError_t launch_scan_tc(const SearchArgs& a, const void* tmaps, int num_sms, cudaStream_t s)
{
    if (a.d == 128) return a.W == 2 ? launch_tc<128, 2>(a, tmaps, num_sms, s) : launch_tc<128, 1>(a, tmaps, num_sms, s);
    if (a.d == 64) return a.W == 2 ? launch_tc<64, 2>(a, tmaps, num_sms, s) : launch_tc<64, 1>(a, tmaps, num_sms, s);
    return cudaErrorInvalidValue;
}

}  // namespace st
