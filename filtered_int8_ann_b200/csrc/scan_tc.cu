// Dense-unit list scan on the 5th-generation tensor cores.
//
// Same method as the warp scan (scan.cu): inside every probed list, the Bloom
// test (sig & mask) == mask decides eligibility, only eligible items are
// scored by the int8 inner product, and the scores feed the final top-k
// (SilverTorch: Index as Model, section on redesigning each stage as a pure
// PyTorch module, Bloom index filter and fused Int8 ANN paragraphs). When many
// queries probe the same list, a unit (512 rows x up to 64 of those queries)
// is a dense int8 contraction, and it runs here as tensor-core tiles instead
// of per-pair dp4a:
//   * the unit's signature bit-planes (the union of its queries' mask bits)
//     are copied by cp.async and tested: pass words [32-row block][query];
//   * rows: a 32-row block with many survivors (for any of the unit's
//     queries) is copied whole by a TMA tile load; a block with few has only
//     its survivors' rows gathered by cp.async; blocks without survivors are
//     not read. Both land in the canonical 128-byte (d = 128) or 64-byte
//     (d = 64) swizzled K-major layout;
//   * one thread issues tcgen05.mma kind::i8 (M = 128 rows, N = the unit's
//     queries rounded up to 16, K = 32) into int32 accumulators in TMEM, one
//     128-row block at a time, and commits to an mbarrier;
//   * epilogue: each thread reads its row's scores from TMEM (tcgen05.ld),
//     applies the pass bits, and keeps a key only if its score reaches the
//     query's running bound (below); kept keys are counted per query, slots
//     are reserved with one atomic per query, and the keys are written.
// Two pipeline stages (operands in shared memory, accumulators in TMEM): the
// rows of unit i load while unit i-1's epilogue runs.
//
// Running top-k bound. Intermediate results should stay on chip (Andromeda
// review, section on why the bottleneck moved from compute to bandwidth), so
// keys that can no longer enter a query's top-k are not written at all. Every
// written key is a real candidate, so if at least k written keys have scores
// >= T, the query's k-th best score is >= T and any key below T can be
// dropped. Each query's written keys are counted in 64 bins over its possible
// score range [-S, S], S = 128 sum_j |q_j| (bin b holds scores in
// [-S + b 2^sh, -S + (b+1) 2^sh)); after a unit, the bins' totals give the
// highest bin edge with k written keys at or above it, published with
// atomicMax. The bound only grows and the final top-k is unchanged (exact).
// With deletions or exclude masks the post-filter is applied before a key is
// counted, so every counted key is still a result candidate.
//
// Waits are bounded: a wait that runs out sets an error bit, the CTA stops,
// waits (bounded) for its copies and MMAs in flight and frees its TMEM.
#include "tc_ptx.cuh"

namespace st {

constexpr int kTcThreads = 128;
constexpr int kTcRows = kWarpItems;   // rows per unit
constexpr int kTcPlaneSlots = 48;     // planes one stage's buffer holds
#ifndef ST_TC_DENSE_BLK
#define ST_TC_DENSE_BLK 24
#endif
constexpr int kTcDenseBlk = ST_TC_DENSE_BLK;  // survivors of a 32-row block from which the whole block is loaded
constexpr uint32_t kTcWaitLimit = 1u << 22;
constexpr int kTcTmemCols = 512;      // 2 stages x 4 row blocks x kTcQMax columns
constexpr size_t kTcMinSmem = 120 * 1024;  // keeps one CTA per SM (it holds all TMEM columns)

struct TcMeta {                       // one unit's data, from its load to its epilogue
    int4 e;                           // {first row, plane block, first slot, rows << 16 | queries}
    int32_t qid[kTcQMax];
    uint32_t pass[16][kTcQMax];       // [32-row block][query] Bloom pass words
    uint32_t uni[16];                 // OR over the queries of the pass words
    unsigned long long up[2][2];      // union of the queries' masks, per warp 0 / 1
    uint8_t tab[kMaskBitsMax];        // signature bit -> plane slot
    int32_t held;                     // planes in the stage buffer (-1: the test reads global planes)
    uint32_t mbmask;                  // 128-row blocks with survivors (MMAs issued for them)
};

struct TcEpi {                        // epilogue scratch of the unit being finished
    uint32_t thr[kTcQMax];            // running bound (biased score) when the unit started
    int32_t qbase[kTcQMax];
    int32_t qsh[kTcQMax];
    uint32_t cnt[kTcQMax], cur[kTcQMax], gbase[kTcQMax];
    uint32_t smax[kTcQMax], smin[kTcQMax];
    uint32_t hist[kTcQMax][kTcBins];
};

template <int D>
__device__ __forceinline__ uint32_t swz(int r, int c)
{
    // canonical swizzled K-major layout: 8-row atoms of 8 * D bytes; the
    // 16-byte chunk c of row r is XORed with the row's place in the atom
    const int x = D == 128 ? (r & 7) : ((r & 7) >> 1);
    return uint32_t((r >> 3) * (8 * D) + (r & 7) * D + ((c ^ x) << 4));
}

template <int D>
__host__ __device__ constexpr size_t tc_dyn_smem()
{
    return size_t(2) * kTcRows * D + size_t(2) * kTcQMax * D + size_t(2) * kTcPlaneSlots * 64 + 1024;
}

template <int D, int W>
__global__ void __launch_bounds__(kTcThreads, 1)
scan_tc_kernel(SearchArgs a, const __grid_constant__ CUtensorMap tmap)
{
    dep_enter();
    const int n_units = a.ctl->n_dense < a.max_units ? a.ctl->n_dense : a.max_units;
    if (int(blockIdx.x) >= n_units) return;  // CTA-uniform, before any allocation

    extern __shared__ unsigned char smem_raw[];
    __shared__ TcMeta meta[3];
    __shared__ TcEpi ep;
    __shared__ __align__(8) uint64_t rows_bar[2];
    __shared__ __align__(8) uint64_t mma_bar[2];
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;

    constexpr int NPL = 64 * W;        // planes per chunk
    constexpr int CH = D / 16;         // 16-byte chunks per row
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t raw_sa = smem_u32(smem_raw);
    unsigned char* const base = smem_raw + (((raw_sa + 1023u) & ~1023u) - raw_sa);
    unsigned char* const Abuf = base;                                   // [2][kTcRows * D]
    unsigned char* const Bbuf = base + 2 * kTcRows * D;                 // [2][kTcQMax * D]
    uint32_t* const Pbuf = reinterpret_cast<uint32_t*>(Bbuf + 2 * kTcQMax * D);  // [2][kTcPlaneSlots][16]

    if (tid == 0) {
        mbar_init(&rows_bar[0], 1);
        mbar_init(&rows_bar[1], 1);
        mbar_init(&mma_bar[0], 1);
        mbar_init(&mma_bar[1], 1);
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async_smem();
    }
    if (warp == 0) {
        tmem_alloc(&s_tmem, kTcTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    const int n_iter = (n_units - int(blockIdx.x) + int(gridDim.x) - 1) / int(gridDim.x);
    const bool filt = a.dead != nullptr || a.qexclude != nullptr;

    // ---- a unit's query slots and mask union -> meta[m] -------------------
    auto load_slots = [&](int m, int it) {
        const int4 e = a.units_tc[blockIdx.x + int64_t(it) * gridDim.x];
        const int qn = e.w & 0xFFFF;
        unsigned long long x = 0, y = 0;
        if (tid < qn) {
            const int qid = a.qlist[e.z + tid];
            meta[m].qid[tid] = qid;
            const ulonglong2 mk = reinterpret_cast<const ulonglong2*>(a.qmask_slot)[e.z + tid];
            x = mk.x;
            y = mk.y;
        }
        if (tid < 64) {  // warps 0 and 1: the union of their queries' masks
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                x |= __shfl_xor_sync(0xffffffffu, x, off);
                y |= __shfl_xor_sync(0xffffffffu, y, off);
            }
            if (lane == 0) {
                meta[m].up[warp][0] = x;
                meta[m].up[warp][1] = y;
            }
        }
        if (tid >= 64 && tid < 80) meta[m].uni[tid - 64] = 0;
        if (tid == 0) {
            meta[m].e = e;
            meta[m].mbmask = 0;
        }
    };

    // ---- request the unit's planes into stage buffer p (after a barrier) ---
    auto request_planes = [&](int m, int p) {
        const unsigned long long u0 = meta[m].up[0][0] | meta[m].up[1][0];
        const unsigned long long u1 = W > 1 ? (meta[m].up[0][1] | meta[m].up[1][1]) : 0ull;
        const int n0 = __popcll(u0);
        const int nb = n0 + __popcll(u1);
        if (nb > kTcPlaneSlots) {
            if (tid == 0) meta[m].held = -1;
            return;
        }
        if (tid < 64 * W) {  // signature bit tid -> its slot
            const unsigned long long word = tid < 64 ? u0 : u1;
            const int bb = tid & 63;
            const unsigned long long below = bb ? (word & ((1ull << bb) - 1ull)) : 0ull;
            meta[m].tab[tid] = uint8_t((tid < 64 ? 0 : n0) + __popcll(below));
        }
        if (tid == 0) meta[m].held = nb;
        const int chunk = meta[m].e.y;
        uint32_t* dst = Pbuf + p * kTcPlaneSlots * 16;
        for (int item = tid; item < 4 * nb; item += kTcThreads) {
            int j = item >> 2;
            const int qq = item & 3;
            // the j-th set bit of the union
            int bit;
            const int c0 = __popc(uint32_t(u0)), c1 = __popc(uint32_t(u0 >> 32)), c2 = __popc(uint32_t(u1));
            if (j < c0) bit = __fns(uint32_t(u0), 0, j + 1);
            else if ((j -= c0) < c1) bit = 32 + __fns(uint32_t(u0 >> 32), 0, j + 1);
            else if ((j -= c1) < c2) bit = 64 + __fns(uint32_t(u1), 0, j + 1);
            else bit = 96 + __fns(uint32_t(u1 >> 32), 0, j - c2 + 1);
            cp_async16_cg(dst + (item >> 2) * 16 + qq * 4, a.planes + (int64_t(chunk) * NPL + bit) * 16 + qq * 4);
        }
    };

    // ---- Bloom test of meta[m] with stage buffer p -------------------------
    auto test_unit = [&](int m, int p) {
        const int4 e = meta[m].e;
        const int qn = e.w & 0xFFFF, len = e.w >> 16;
        const int held = meta[m].held;
        const int w = tid & 15;
        const uint32_t valid = len >= 32 * (w + 1) ? 0xFFFFFFFFu : (len <= 32 * w ? 0u : ((1u << (len - 32 * w)) - 1u));
        const uint32_t* pl = Pbuf + p * kTcPlaneSlots * 16;
        const uint32_t* gpl = a.planes + int64_t(e.y) * NPL * 16;
        for (int j = 0; j < kTcQMax / 8; ++j) {
            const int qs = (tid >> 4) + 8 * j;  // this half-warp's query
            uint32_t acc = 0;
            int qid = 0;
            if (qs < qn) {
                qid = meta[m].qid[qs];
                const int nb = __ldg(a.qnbits + qid);
                const uint8_t* bits = a.qbits + int64_t(qid) * kMaskBitsMax;
                acc = 0xFFFFFFFFu;
                if (held >= 0) {
                    for (int i = 0; i < nb; ++i) acc &= pl[meta[m].tab[__ldg(bits + i)] * 16 + w];
                } else {
                    for (int i = 0; i < nb; ++i) acc &= __ldg(gpl + __ldg(bits + i) * 16 + w);
                }
                acc &= valid;
                meta[m].pass[w][qs] = acc;
                if (acc) atomicOr(&meta[m].uni[w], acc);
            }
            uint32_t c = __popc(acc);
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
            if (qs < qn && w == 0 && c)
                atomicAdd(&a.eligible_cnt[int64_t(qid) * (kCntStride / 2)], (unsigned long long)c);
        }
    };

    // ---- issue the row and query copies of meta[m] into operand stage s ----
    auto issue_rows = [&](int m, int s) {
        const int4 e = meta[m].e;
        const int qn = e.w & 0xFFFF;
        unsigned char* A = Abuf + s * kTcRows * D;
        unsigned char* Bq = Bbuf + s * kTcQMax * D;
        uint32_t mb = 0, dense_bytes = 0;
        uint32_t dmask = 0;  // 32-row blocks loaded whole
#pragma unroll
        for (int b = 0; b < 16; ++b) {
            const int pc = __popc(meta[m].uni[b]);
            if (pc) mb |= 1u << (b >> 2);
            if (pc >= kTcDenseBlk) {
                dmask |= 1u << b;
                dense_bytes += 32 * D;
            }
        }
        if (tid == 0) {
            meta[m].mbmask = mb;
            mbar_arrive_expect_tx(&rows_bar[s], dense_bytes);
            for (int b = 0; b < 16; ++b)
                if ((dmask >> b) & 1u) tma_load_2d(A + b * 32 * D, &tmap, 0, e.x + 32 * b, &rows_bar[s]);
        }
        // the survivors of the other blocks, one lane per row
        for (int b = warp; b < 16; b += 4) {
            const uint32_t u = meta[m].uni[b];
            if (((dmask >> b) & 1u) || !((u >> lane) & 1u)) continue;
            const int r = 32 * b + lane;
            const int8_t* src = a.items + (int64_t(e.x) + r) * D;
#pragma unroll
            for (int c = 0; c < CH; ++c) cp_async16_cg(A + swz<D>(r, c), src + 16 * c);
        }
        // the unit's query vectors (rows past qn are never read back)
        for (int item = tid; item < qn * CH; item += kTcThreads) {
            const int q = item / CH, c = item - q * CH;
            cp_async16(Bq + swz<D>(q, c), a.queries + int64_t(meta[m].qid[q]) * D + 16 * c);
        }
    };

    // ---- tensor-core MMAs of operand stage s (one thread) ------------------
    auto issue_mma = [&](int m, int s) {
        const int qn = meta[m].e.w & 0xFFFF;
        const int N = (qn + 15) & ~15;
        const uint32_t idesc = idesc_i8(128, N);
        const uint32_t a0 = smem_u32(Abuf + s * kTcRows * D), b0 = smem_u32(Bbuf + s * kTcQMax * D);
        const uint32_t mbm = meta[m].mbmask;
        tc_fence_after();
        for (int mb = 0; mb < 4; ++mb) {
            if (!((mbm >> mb) & 1u)) continue;
#pragma unroll
            for (int ks = 0; ks < D / 32; ++ks)
                tc_mma_i8(tmem + uint32_t(s * 256 + mb * kTcQMax), smem_desc_kmajor(a0 + mb * 128 * D + ks * 32, D),
                          smem_desc_kmajor(b0 + ks * 32, D), idesc, ks > 0 ? 1u : 0u);
        }
        tc_commit(&mma_bar[s]);
    };

    // ---- epilogue of meta[m] whose accumulators are in TMEM stage s --------
    // Returns false when the wait for its MMAs ran out.
    uint32_t mph = 0;  // parity of the next wait on mma_bar[s], bit s
    auto epilogue = [&](int m, int s) -> bool {
        const uint32_t mbm = meta[m].mbmask;
        if (mbm == 0u) return true;  // no survivors: no MMA was issued
        const bool ok = mbar_wait(&mma_bar[s], (mph >> s) & 1u, kTcWaitLimit);
        mph ^= 1u << s;
        tc_fence_after();
        const int4 e = meta[m].e;
        const int qn = e.w & 0xFFFF;
        if (tid < qn) {
            const int qid = meta[m].qid[tid];
            ep.thr[tid] = __ldcg(a.score_rng + int64_t(qid) * kCntStride + kRngThr);
            const int2 sc = a.qscale[qid];
            ep.qbase[tid] = sc.x;
            ep.qsh[tid] = sc.y;
            ep.cnt[tid] = 0;
            ep.cur[tid] = 0;
            ep.smax[tid] = 0;
            ep.smin[tid] = 0;
        }
        {
            uint4* h = reinterpret_cast<uint4*>(&ep.hist[0][0]);
            for (int i = tid; i < qn * kTcBins / 4; i += kTcThreads) h[i] = make_uint4(0, 0, 0, 0);
        }
        if (__syncthreads_or(!ok)) return false;
        const int nsl = (qn + 15) >> 4;
        // pass 1: count the keys at or above the bound, per query and bin
        bool anyk = false;
        for (int mb = 0; mb < 4; ++mb) {
            if (!((mbm >> mb) & 1u)) continue;
            const int r = mb * 128 + warp * 32 + lane;
            const int wb = r >> 5;
            for (int sl = 0; sl < nsl; ++sl) {
                uint32_t v[16];
                tmem_ld16(tmem + (uint32_t(warp * 32) << 16) + uint32_t(s * 256 + mb * kTcQMax + sl * 16), v);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int q = sl * 16 + j;
                    if (q >= qn || !((meta[m].pass[wb][q] >> lane) & 1u)) continue;
                    const int32_t score = int32_t(v[j]);
                    const uint32_t ub = uint32_t(score) ^ 0x80000000u;
                    if (ub < ep.thr[q]) continue;
                    if (filt && !keep_item(a, meta[m].qid[q], int64_t(e.x) + r)) continue;
                    anyk = true;
                    atomicAdd(&ep.cnt[q], 1u);
                    atomicAdd(&ep.hist[q][(score - ep.qbase[q]) >> ep.qsh[q]], 1u);
                    atomicMax(&ep.smax[q], ub);
                    atomicMax(&ep.smin[q], ~ub);
                }
            }
        }
        __syncthreads();
        if (tid < qn && ep.cnt[tid]) {
            const int qid = meta[m].qid[tid];
            ep.gbase[tid] = atomicAdd(&a.cand_cnt[int64_t(qid) * kCntStride], ep.cnt[tid]);
            atomicMax(&a.score_rng[int64_t(qid) * kCntStride], ep.smax[tid]);
            atomicMax(&a.score_rng[int64_t(qid) * kCntStride + 1], ep.smin[tid]);
        }
        __syncthreads();
        // pass 2: write the same keys into the reserved slots
        if (__any_sync(0xffffffffu, anyk)) {
            for (int mb = 0; mb < 4; ++mb) {
                if (!((mbm >> mb) & 1u)) continue;
                const int r = mb * 128 + warp * 32 + lane;
                const int wb = r >> 5;
                const uint32_t id = uint32_t(e.x + r);
                for (int sl = 0; sl < nsl; ++sl) {
                    uint32_t v[16];
                    tmem_ld16(tmem + (uint32_t(warp * 32) << 16) + uint32_t(s * 256 + mb * kTcQMax + sl * 16), v);
                    tmem_wait_ld();
                    if (!anyk) continue;
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int q = sl * 16 + j;
                        if (q >= qn || !((meta[m].pass[wb][q] >> lane) & 1u)) continue;
                        const int32_t score = int32_t(v[j]);
                        const uint32_t ub = uint32_t(score) ^ 0x80000000u;
                        if (ub < ep.thr[q]) continue;
                        const int qid = meta[m].qid[q];
                        if (filt && !keep_item(a, qid, int64_t(id))) continue;
                        const uint32_t pos = ep.gbase[q] + atomicAdd(&ep.cur[q], 1u);
                        if (int64_t(pos) < a.cap) a.cand[int64_t(qid) * a.cap + pos] = pack_key(score, id);
                    }
                }
            }
        }
        // publish the counts and raise each query's bound: the highest bin
        // edge with at least k written keys at or above it
        for (int q0 = 0; q0 < qn; q0 += 4 * 4) {
            uint32_t g[4][2];
            int qq[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                qq[t] = q0 + warp + 4 * t;
                g[t][0] = g[t][1] = 0;
                if (qq[t] < qn && ep.cnt[qq[t]]) {
                    uint32_t* gh = a.tc_hist + int64_t(meta[m].qid[qq[t]]) * kTcBins;
                    const uint32_t c0 = ep.hist[qq[t]][2 * lane], c1 = ep.hist[qq[t]][2 * lane + 1];
                    g[t][0] = c0 ? atomicAdd(gh + 2 * lane, c0) + c0 : __ldcg(gh + 2 * lane);
                    g[t][1] = c1 ? atomicAdd(gh + 2 * lane + 1, c1) + c1 : __ldcg(gh + 2 * lane + 1);
                }
            }
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                if (qq[t] >= qn || !ep.cnt[qq[t]]) continue;  // warp-uniform
                uint32_t incl = g[t][0] + g[t][1];  // suffix sum over lanes >= this one
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const uint32_t o = __shfl_down_sync(0xffffffffu, incl, off);
                    if (lane + off < 32) incl += o;
                }
                const uint32_t kk = uint32_t(a.k);
                uint32_t best = 0;  // highest bin b with (keys in bins >= b) >= k
                if (incl - g[t][0] >= kk) best = uint32_t(2 * lane + 1);
                else if (incl >= kk) best = uint32_t(2 * lane);
                best = __reduce_max_sync(0xffffffffu, best);
                if (lane == 0 && best > 0) {
                    const int32_t T = ep.qbase[qq[t]] + int32_t(best << ep.qsh[qq[t]]);
                    atomicMax(a.score_rng + int64_t(meta[m].qid[qq[t]]) * kCntStride + kRngThr,
                              uint32_t(T) ^ 0x80000000u);
                }
            }
        }
        tc_fence_before();
        return true;
    };

    // ---- pipeline ------------------------------------------------------------
    load_slots(0, 0);
    __syncthreads();
    request_planes(0, 0);
    cp_async_commit();
    bool aborted = false;
    for (int it = 0; it < n_iter; ++it) {
        const int s = it & 1, m = it % 3;
        const bool has_next = it + 1 < n_iter;
        // next unit: slots, then its planes (into the other plane buffer)
        if (has_next) load_slots((it + 1) % 3, it + 1);
        if (has_next) cp_async_wait_group<0>();  // this unit's planes
        __syncthreads();
        if (has_next) request_planes((it + 1) % 3, (it + 1) & 1);
        cp_async_commit();
        if (!has_next) cp_async_wait_group<0>();
        __syncthreads();
        test_unit(m, s);
        __syncthreads();
        issue_rows(m, s);
        cp_async_commit();
        // the previous unit's epilogue overlaps these copies
        if (it > 0 && !epilogue((it - 1) % 3, s ^ 1)) {
            aborted = true;
            break;
        }
        cp_async_wait_group<0>();
        fence_proxy_async_smem();
        if (tid == 0 && !mbar_wait(&rows_bar[s], uint32_t(it >> 1) & 1u, kTcWaitLimit)) s_abort = 1;
        __syncthreads();
        if (s_abort) {
            aborted = true;
            break;
        }
        if (tid == 0 && meta[m].mbmask) issue_mma(m, s);
    }
    if (!aborted && n_iter > 0 && !epilogue((n_iter - 1) % 3, (n_iter - 1) & 1)) aborted = true;

    // teardown: nothing of this CTA may be in flight when its TMEM is freed
    cp_async_wait_all();
    if (aborted) {
        if (tid == 0) {
            set_error(a.err, kErrTcWait);
            for (int st2 = 0; st2 < 2; ++st2) {
                mbar_wait(&rows_bar[st2], 0, 1u << 12);
                mbar_wait(&mma_bar[st2], (mph >> st2) & 1u, 1u << 12);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTcTmemCols);
}

bool scan_tc_supported(int d) { return d == 64 || d == 128; }

template <int D, int W>
static cudaError_t launch_tc(const SearchArgs& a, const void* tmap, int num_sms, cudaStream_t s)
{
    size_t smem = tc_dyn_smem<D>();
    if (smem < kTcMinSmem) smem = kTcMinSmem;
    const void* fn = reinterpret_cast<const void*>(scan_tc_kernel<D, W>);
    cudaError_t e = ensure_smem_attr(fn, int(smem));
    if (e != cudaSuccess) return e;
    CUtensorMap map;
    memcpy(&map, tmap, sizeof(map));
    return launch_dep(scan_tc_kernel<D, W>, dim3(num_sms), dim3(kTcThreads), smem, s, a, map);
}

cudaError_t launch_scan_tc(const SearchArgs& a, const void* tmap, int num_sms, cudaStream_t s)
{
    if (a.d == 128) return a.W == 2 ? launch_tc<128, 2>(a, tmap, num_sms, s) : launch_tc<128, 1>(a, tmap, num_sms, s);
    if (a.d == 64) return a.W == 2 ? launch_tc<64, 2>(a, tmap, num_sms, s) : launch_tc<64, 1>(a, tmap, num_sms, s);
    return cudaErrorInvalidValue;
}

}  // namespace st
