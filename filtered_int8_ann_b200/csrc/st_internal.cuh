// Internal definitions shared by the libst kernels and the host API.
#pragma once
#include <utility>

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/st.h"

namespace st {

// ----------------------------------------------------------------------------
// Tunables
// ----------------------------------------------------------------------------
constexpr int kScanBlock = 128;            // threads per scan CTA (four warps sharing a unit counter)
constexpr int kWarpItems = 512;            // list rows per work unit (one warp)
constexpr int kQMax = 16;                  // queries per work unit
// Dense units: lists probed by at least tc_min_q queries go to the tensor-core
// scan in units of up to kTcQMax queries (the MMA's N).
constexpr int kTcQMax = 32;
constexpr int kTcMinQDefault = 8;
constexpr int kSelSample = 512;             // index rows whose signatures estimate each query's selectivity
constexpr int kSelMinProbes = 2048;         // (query, list) probes from which selectivity routes lists
constexpr int kTcBins = 1024;              // per-query score bins of the written candidate keys
constexpr int kRngThr = 12;                // score_rng word: the query's running score bound (biased)

constexpr int kProbeBlock = 512;
constexpr int kProbeSmemKeys = 16384;      // nlist up to this keeps probe keys in smem
constexpr int kSelectBlock = 1024;
// Per-query counters sit one 128-byte line apart, so the reservation atomics
// of different queries spread over the L2 slices instead of queueing on one.
constexpr int kCntStride = 32;             // uint32 words (16 uint64) per query

// Row stride (keys) of the search probe's [B][nlist] centroid keys: even, so
// every row starts on a 16-byte boundary for vector copies.
__host__ __device__ __forceinline__ int64_t probe_keys_ld(int nlist) { return (int64_t(nlist) + 1) & ~int64_t(1); }
constexpr int kMaskBitsMax = 128;          // signature bits
constexpr int kSlotBits = 32;              // mask bits a slot carries (the rest: the query's own list)
constexpr int kSelBits = 11;               // radix digit of the selections
constexpr int kSelBins = 1 << kSelBits;
constexpr int kSelTieCap = 4096;           // cut-bin keys the final top-k keeps per query

// Device error word bits (st_index_check reports any of them as ST_ERR_DEVICE).
enum : uint32_t {
    kErrUnitDecode = 1u << 0,   // a work unit did not map to a list
    kErrSelectCount = 1u << 2,  // a selection collected the wrong number of keys
    kErrOverflowPath = 1u << 3, // the exact overflow path met an impossible state
    kErrUnitTable = 1u << 4,    // more work units than the host-sized table holds
    kErrUpdateId = 1u << 6,     // an in-place update named a row outside the index
    kErrTcWait = 1u << 7,       // a wait of the tensor-core scan ran out (bounded wait expired)
};

// ----------------------------------------------------------------------------
// 64-bit ranking key: larger key = better (score descending, then id ascending)
//   high 32 bits: score with the sign bit flipped (order-preserving unsigned)
//   low  32 bits: 0xFFFFFFFF - id
// Key 0 decodes to (score INT32_MIN, id -1): the padding value. Real scores are
// bounded by d * 128 * 128 <= 2^23, so a real key is never 0.
// ----------------------------------------------------------------------------
__host__ __device__ __forceinline__ uint64_t pack_key(int32_t score, uint32_t id)
{
    return (uint64_t(uint32_t(score) ^ 0x80000000u) << 32) | uint64_t(0xFFFFFFFFu - id);
}
__host__ __device__ __forceinline__ int32_t key_score(uint64_t key)
{
    return int32_t(uint32_t(key >> 32) ^ 0x80000000u);
}
__host__ __device__ __forceinline__ int64_t key_id(uint64_t key)
{
    return int64_t(int32_t(0xFFFFFFFFu - uint32_t(key)));
}

// ----------------------------------------------------------------------------
// Per-search state
// ----------------------------------------------------------------------------
struct PlanCtl {
    int32_t n_units;       // work units allocated by the plan (clamped to the table by the scan)
    int32_t n_dense;       // dense (tensor-core) units allocated by the plan
    int32_t max_qsel;      // the batch's largest sample count of one query (selectivity routing)
    int32_t pad;
};

struct SearchArgs {
    // index (read-only)
    const int8_t* items;
    const uint64_t* sigs;
    const uint32_t* planes;      // [n_plane_chunks][64W][16] signature bit-planes, one block per chunk
    const int4* chunk_desc;      // [n_chunks] the chunks (up to kWarpItems rows of one list), list by list:
                                 // {first row, plane block, rows, list}
    const int32_t* chunk_start;  // [nlist+1] first chunk_desc entry of each list
    int32_t n_chunks;
    int32_t n_plane_chunks;      // plane blocks allocated
    int64_t n_rows;              // rows the item and signature arrays hold
    const int8_t* centroids;
    int32_t d, nlist, W;
    // request
    const int8_t* queries;
    const uint64_t* qmasks;
    int32_t B, P, k;
    // outputs
    int64_t* out_ids;
    int32_t* out_scores;
    int64_t* out_eligible;   // may be null
    int64_t* out_cands;      // may be null: candidate keys written per query
    // scratch (the zeroed block first: one memset clears it)
    int32_t* list_cnt;       // [nlist] queries filed into each list      (zeroed)
    int32_t* probe_done;     // [B] probe slices finished per query       (zeroed)
    uint32_t* cand_cnt;      // [B][kCntStride] candidates reserved per query, word 0 used (zeroed)
    uint32_t* score_rng;     // [B][kCntStride] per-query words of the final top-k and the dense
                             // scan's running bound (zeroed)
    uint32_t* sel_hist;      // [B][kSelBins] final top-k: candidate score histogram (zeroed)
    uint32_t* sel_cursor;    // [B][kSelBins] final top-k: keys placed per bin (zeroed)
    uint64_t* sel_out;       // [B][k] final top-k: keys above the cut, grouped by bin
    uint64_t* sel_tie;       // [B][kSelTieCap] final top-k: keys of the cut bin
    int64_t id_offset;       // added to every returned item id
    const uint32_t* dead;    // [ceil(n / 32)] deleted items, or null (none deleted)
    const uint64_t* qexclude;  // [B][W] exclude masks, or null
    const uint64_t* or_masks;  // [B][n_or][W] alternative masks (an item passing any mask is eligible), or null
    int32_t n_or;              // alternatives per query besides qmasks (0: none)
    unsigned long long* eligible_cnt;  // [B][kCntStride / 2], word 0 used        (zeroed)
    PlanCtl* ctl;            // unit allocation counter                   (zeroed)
    int32_t* probe;          // [B][P]
    uint64_t* probe_keys;    // [B][nlist] when a probe slice does not fit shared memory, else null
    uint64_t* probe_part;    // [B][S][P] best keys of each probe slice
    int32_t* list_ustart;    // [nlist] first unit of each probed list
    int32_t* qlist;          // [nlist][B] slot row of each list: ids of the queries probing it
    uint64_t* qmask_slot;    // [nlist][B][2] that query's mask words (word 1 = 0 when W = 1)
    uint8_t* slot_bits;      // [nlist][B][kSlotBits] that query's first kSlotBits mask bits, increasing
    uint8_t* qbits;          // [B][1 + n_or][kMaskBitsMax] each mask's bits, in increasing order
    int32_t* qnbits;         // [B][1 + n_or] number of bits of each mask
    int4* units;             // [max_units] {first row, chunk, first slot, rows << 16 | queries}
    int4* units_tc;          // [max_units] dense units, same entries (up to kTcQMax queries)
    int32_t max_units;
    int32_t tc_min_q;        // queries per list from which its units are dense (0: no dense units)
    const uint64_t* sig_sample;  // [n_sample][W] signatures of evenly spaced rows of the index
    int32_t n_sample;
    uint16_t* qsel;          // [B] sample rows passing each query's mask(s), or null (no selectivity routing)
    int2* qscale;            // [B] per query {lowest possible score -S, shift of kTcBins bins over
                             // [-S, S]}: S = 128 sum_j |q_j| bounds |<q, x>| for any int8 row x
    uint32_t* qhist;         // [B][kTcBins] candidate keys written by the scans per score bin (zeroed)
    int32_t count_bins;      // the warp scan counts its keys in qhist (the final top-k reads them)
    uint64_t* cand;          // [B][cap]
    int64_t cap;             // candidate keys per query
    uint32_t* err;           // device error word
};


// A list's units go to the tensor-core scan when enough queries probe it.
__device__ __forceinline__ bool dense_list(const SearchArgs& a, int cnt)
{
    return a.tc_min_q > 0 && cnt >= a.tc_min_q;
}

// A list probed by fewer queries still goes to the tensor cores when they
// expect together at least 3/4 of an eligible (query, row) pair per row (each
// query's expectation: the share of a fixed sample of the index's rows that
// passes its mask). Such a list's tiles waste little, while the warp scan
// would score and write nearly every row once per query. Only the choice of
// scan depends on it, never the result.
__device__ __forceinline__ bool dense_by_selectivity(const SearchArgs& a, int L, int cnt)
{
    if (a.qsel == nullptr || a.n_sample <= 0) return false;
    const uint32_t need = 3u * uint32_t(a.n_sample);
    if (4u * uint32_t(cnt) * uint32_t(a.ctl->max_qsel) < need) return false;  // not even with cnt of the best query
    uint32_t s = 0;
    for (int i = 0; i < cnt && 4u * s < need; ++i) s += a.qsel[a.qlist[int64_t(L) * a.B + i]];
    return 4u * s >= need;
}

// Programmatic dependent launch: launch_dep() lets a kernel start while its
// predecessor in the stream drains; every such kernel calls dep_enter() first
// (wait for the predecessor's completion and memory, then let its own
// successor launch).
__device__ __forceinline__ void dep_enter()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_dep(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args&&... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ----------------------------------------------------------------------------
// Small device helpers
// ----------------------------------------------------------------------------
__device__ __forceinline__ int32_t dot16(const int4 a, const int4 b, int32_t acc)
{
    acc = __dp4a(a.x, b.x, acc);
    acc = __dp4a(a.y, b.y, acc);
    acc = __dp4a(a.z, b.z, acc);
    acc = __dp4a(a.w, b.w, acc);
    return acc;
}

__device__ __forceinline__ void set_error(uint32_t* err, uint32_t bit) { atomicOr(err, bit); }

// Count one key in bin `bin` of `hist` for every lane of `members` (the lanes
// that call it, all of them): lanes with the same bin add once together.
__device__ __forceinline__ void count_bin(uint32_t* hist, int bin, unsigned members)
{
    const unsigned same = __match_any_sync(members, bin);
    if ((threadIdx.x & 31) == __ffs(same) - 1) atomicAdd(hist + bin, uint32_t(__popc(same)));
}

__device__ __forceinline__ unsigned lanemask_lt()
{
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte asynchronous copy global -> shared (cp.async, L1-allocating)
__device__ __forceinline__ void cp_async16(void* dst, const void* src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
// 16-byte asynchronous copy global -> shared that bypasses L1 (data read once)
__device__ __forceinline__ void cp_async16_cg(void* dst, const void* src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// Wait until at most N of this thread's committed cp.async groups are pending.
template <int N>
__device__ __forceinline__ void cp_async_wait_group()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ----------------------------------------------------------------------------
// Block-wide selection (one CTA of BLOCK threads)
// ----------------------------------------------------------------------------
struct SelectSmem {
    uint32_t hist[kSelBins];
    uint32_t hist2[kSelBins];
    uint32_t part[32];
    unsigned long long red_lo[32], red_hi[32];
    uint64_t prefix;     // high bits of the threshold fixed so far
    int64_t krem;        // rank still to find below the prefix
    int32_t shift;       // bits below the prefix
    int32_t done;
    int32_t found;
    int32_t count;
    uint32_t lo32, hi32, maxcnt;
};

// Block exclusive scan of one value per thread; `total` gets the block sum.
template <int BLOCK>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* part, uint32_t& total)
{
    constexpr int NW = BLOCK / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += t;
    }
    if (lane == 31) part[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = lane < NW ? part[lane] : 0u;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += t;
        }
        if (lane < NW) part[lane] = w;
    }
    __syncthreads();
    const uint32_t before = warp > 0 ? part[warp - 1] : 0u;
    total = part[NW - 1];
    __syncthreads();
    return before + incl - v;
}

// A threshold T such that exactly k of the n unique keys are >= T (1 <= k <= n).
// MSB-first radix select restricted to the bits where the keys differ (the
// score's high bits are shared by all candidates), 11-bit digits (2048 shared
// bins, so plain shared atomics rarely collide), and an early exit as soon as
// the bucket holding the k-th key is taken whole. `keys` may be shared or
// global memory.
template <int BLOCK>
__device__ uint64_t block_select_threshold(const uint64_t* keys, int64_t n, int64_t k, SelectSmem& s,
                                           uint32_t* err)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int NW = BLOCK / 32;
    uint64_t lo = ~0ull, hi = 0ull;
    for (int64_t i = tid; i < n; i += BLOCK) {
        const uint64_t x = keys[i];
        lo = x < lo ? x : lo;
        hi = x > hi ? x : hi;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const uint64_t a = __shfl_xor_sync(0xffffffffu, lo, off), b = __shfl_xor_sync(0xffffffffu, hi, off);
        lo = a < lo ? a : lo;
        hi = b > hi ? b : hi;
    }
    if (lane == 0) {
        s.red_lo[warp] = lo;
        s.red_hi[warp] = hi;
    }
    __syncthreads();
    if (warp == 0) {
        lo = lane < NW ? s.red_lo[lane] : ~0ull;
        hi = lane < NW ? s.red_hi[lane] : 0ull;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const uint64_t a = __shfl_xor_sync(0xffffffffu, lo, off), b = __shfl_xor_sync(0xffffffffu, hi, off);
            lo = a < lo ? a : lo;
            hi = b > hi ? b : hi;
        }
        if (lane == 0) {
            const uint64_t diff = lo ^ hi;
            const int top = diff ? 64 - __clzll(static_cast<long long>(diff)) : 0;
            s.prefix = top >= 64 ? 0ull : (hi >> top) << top;
            s.shift = top;
            s.krem = k;
            s.done = (top == 0);
            if (top == 0) s.prefix = hi;
        }
    }
    __syncthreads();
    // at most ceil(64 / kSelBits) rounds; each round either finishes or fixes
    // kSelBits more bits, so the loop always ends
    for (int round = 0; round < 8 && !s.done; ++round) {
        const int shift_hi = s.shift;
        const int dbits = shift_hi < kSelBits ? shift_hi : kSelBits;
        const int shift = shift_hi - dbits;
        const int nb = 1 << dbits;
        const uint64_t prefix = s.prefix;
        for (int i = tid; i < nb; i += BLOCK) s.hist[i] = 0;
        __syncthreads();
        for (int64_t i = tid; i < n; i += BLOCK) {
            const uint64_t x = keys[i];
            if (shift_hi >= 64 || (x >> shift_hi) == (prefix >> shift_hi))
                atomicAdd(&s.hist[uint32_t(x >> shift) & uint32_t(nb - 1)], 1u);
        }
        __syncthreads();
        // thread t owns `per` bins counted down from the top bin
        const int per = nb >= BLOCK ? nb / BLOCK : 1;
        const int owners = nb / per;
        uint32_t local = 0;
        if (tid < owners)
            for (int j = 0; j < per; ++j) local += s.hist[nb - 1 - (tid * per + j)];
        if (tid == 0) s.found = 0;
        uint32_t total;
        const uint32_t excl = block_excl_scan<BLOCK>(local, s.part, total);
        const int64_t krem = s.krem;
        if (tid < owners && int64_t(excl) < krem && krem <= int64_t(excl) + int64_t(local)) {
            int64_t acc = excl;
            for (int j = 0; j < per; ++j) {
                const int bin = nb - 1 - (tid * per + j);
                const uint32_t c = s.hist[bin];
                if (acc + c >= krem) {
                    const int64_t nk = krem - acc;
                    s.prefix = prefix | (uint64_t(bin) << shift);
                    s.krem = nk;
                    s.shift = shift;
                    s.done = (shift == 0) || (int64_t(c) == nk);
                    s.found = 1;
                    break;
                }
                acc += c;
            }
        }
        __syncthreads();
        if (!s.found) {  // impossible for 1 <= k <= n unique keys: report and stop
            if (tid == 0) {
                set_error(err, kErrSelectCount);
                s.done = 1;
            }
            __syncthreads();
        }
    }
    return s.prefix;
}

// Copy every key >= thr from keys[0..n) into out[] (at most out_cap); returns
// how many keys were >= thr.
template <int BLOCK>
__device__ int32_t block_collect_ge(const uint64_t* keys, int64_t n, uint64_t thr, uint64_t* out,
                                    int32_t out_cap, SelectSmem& s)
{
    if (threadIdx.x == 0) s.count = 0;
    __syncthreads();
    for (int64_t base = 0; base < n; base += BLOCK) {
        const int64_t i = base + threadIdx.x;
        uint64_t key = 0;
        bool take = false;
        if (i < n) {
            key = keys[i];
            take = key >= thr;
        }
        const unsigned bal = __ballot_sync(0xffffffffu, take);
        if (bal) {
            int32_t b0 = 0;
            if ((threadIdx.x & 31) == 0) b0 = atomicAdd(&s.count, __popc(bal));
            b0 = __shfl_sync(0xffffffffu, b0, 0);
            const int32_t pos = b0 + __popc(bal & lanemask_lt());
            if (take && pos < out_cap) out[pos] = key;
        }
    }
    __syncthreads();
    const int32_t count = s.count;
    __syncthreads();  // a following collect may reset the counter at once
    return count;
}

// Sort a[0..m) descending with a bitonic network in shared memory (the keys
// are padded with zeros to a power of two; `a` needs room for next_pow2(m)
// keys). Compact and slow; the counting sort below uses it only as a fallback.
template <int BLOCK>
__device__ void block_bitonic_desc(uint64_t* a, int m)
{
    int mm = 1;
    while (mm < m) mm <<= 1;
    for (int i = m + threadIdx.x; i < mm; i += BLOCK) a[i] = 0;
    __syncthreads();
    for (int size = 2; size <= mm; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = threadIdx.x; i < (mm >> 1); i += BLOCK) {
                const int lo = 2 * i - (i & (stride - 1));
                const int hi = lo + stride;
                const bool desc = (lo & size) == 0;
                const uint64_t x = a[lo], y = a[hi];
                if (desc ? (x < y) : (x > y)) {
                    a[lo] = y;
                    a[hi] = x;
                }
            }
            __syncthreads();
        }
    }
}

// Sort a[0..m) descending, exactly, by counting: a histogram of the keys' high
// words (the biased scores) over kSelBins bins spanning their range gives each
// bin its output segment (keys of higher bins come first); keys are scattered
// into their segments in `tmp`, and each key's place inside its segment is the
// number of keys of the segment greater than it (keys are unique). The segments
// of a top-k are short; when one holds more than 64 keys (for example many
// equal scores) the bitonic network is used instead, which needs room for
// next_pow2(m) keys in `a`. `tmp` needs m keys.
template <int BLOCK>
__device__ void block_sort_desc_counting(uint64_t* a, int m, uint64_t* tmp, SelectSmem& s)
{
    constexpr int NW = BLOCK / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (m <= 1) {
        __syncthreads();
        return;
    }
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
    for (int i = tid; i < m; i += BLOCK) {
        const uint32_t h = uint32_t(a[i] >> 32);
        lo = h < lo ? h : lo;
        hi = h > hi ? h : hi;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, off));
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, off));
    }
    if (lane == 0) {
        s.red_lo[warp] = lo;
        s.red_hi[warp] = hi;
    }
    for (int i = tid; i < kSelBins; i += BLOCK) {
        s.hist[i] = 0;
        s.hist2[i] = 0;
    }
    __syncthreads();
    if (tid == 0) {
        uint32_t l = 0xFFFFFFFFu, h = 0u;
        for (int w = 0; w < NW; ++w) {
            l = min(l, uint32_t(s.red_lo[w]));
            h = max(h, uint32_t(s.red_hi[w]));
        }
        s.lo32 = l;
        s.hi32 = h;
        s.maxcnt = 0;
    }
    __syncthreads();
    const uint32_t base = s.lo32;
    int shift = 0;
    while (((s.hi32 - base) >> shift) >= uint32_t(kSelBins)) ++shift;
    for (int i = tid; i < m; i += BLOCK) atomicAdd(&s.hist[(uint32_t(a[i] >> 32) - base) >> shift], 1u);
    __syncthreads();
    // descending exclusive scan: start of bin b = keys in bins above b
    constexpr int PER = kSelBins / BLOCK > 0 ? kSelBins / BLOCK : 1;
    const int owners = kSelBins / PER;
    uint32_t local = 0, mx = 0;
    if (tid < owners)
        for (int j = 0; j < PER; ++j) {
            const uint32_t c = s.hist[kSelBins - 1 - (tid * PER + j)];
            local += c;
            mx = c > mx ? c : mx;
        }
    uint32_t total;
    uint32_t run = block_excl_scan<BLOCK>(local, s.part, total);
    if (tid < owners)
        for (int j = 0; j < PER; ++j) {
            const int bin = kSelBins - 1 - (tid * PER + j);
            s.hist2[bin] = run;
            run += s.hist[bin];
        }
    if (mx > 64) atomicMax(&s.maxcnt, mx);
    __syncthreads();
    if (s.maxcnt > 64) {
        block_bitonic_desc<BLOCK>(a, m);
        return;
    }
    for (int i = tid; i < m; i += BLOCK) {
        const uint64_t key = a[i];
        const uint32_t bin = (uint32_t(key >> 32) - base) >> shift;
        tmp[atomicAdd(&s.hist2[bin], 1u)] = key;
    }
    __syncthreads();
    for (int p = tid; p < m; p += BLOCK) {
        const uint64_t key = tmp[p];
        const uint32_t bin = (uint32_t(key >> 32) - base) >> shift;
        const int end = int(s.hist2[bin]);
        const int beg = end - int(s.hist[bin]);
        int r = 0;
        for (int j = beg; j < end; ++j) r += tmp[j] > key ? 1 : 0;
        a[beg + r] = key;
    }
    __syncthreads();
}

// ----------------------------------------------------------------------------
// Histogram top-k. The keys' scores are binned over kSelBins bins spanning a
// range [lo, hi] that contains them all: bin = (score - lo) >> sh, sh the
// smallest shift that fits the range. Suffix sums of the bin counts give the
// bin holding the k-th key (the cut bin) and the output segment of every bin
// above it, so the keys of those bins can be scattered straight to their
// segments; only the cut bin's keys need an exact selection, and each key's
// place inside its segment is the number of the segment's keys greater than
// it (very long segments, i.e. many equal or close scores, use the bitonic
// network instead).
// ----------------------------------------------------------------------------
// Candidate post-filter of query q: false for an item that was deleted or
// whose signature holds every bit of q's (non-zero) exclude mask. Local id.
__device__ __forceinline__ bool keep_item(const SearchArgs& a, int q, int64_t id)
{
    if (a.dead && ((a.dead[id >> 5] >> (id & 31)) & 1u)) return false;
    if (a.qexclude) {
        const int W = a.W;
        const uint64_t x0 = a.qexclude[int64_t(q) * W], x1 = W > 1 ? a.qexclude[int64_t(q) * W + 1] : 0ull;
        if (x0 | x1) {
            const uint64_t* sg = a.sigs + id * W;
            if ((sg[0] & x0) == x0 && (W < 2 || (sg[1] & x1) == x1)) return false;
        }
    }
    return true;
}

struct TopkCut {
    int32_t lo;     // range base
    uint32_t sh;    // bin shift
    int cut;        // cut bin (-1: n <= k, every key is taken)
    int above;      // keys in the bins above the cut
    int tcount;     // keys in the cut bin
    int m;          // min(n, k)
    int maxseg;     // longest output segment
};

__host__ __device__ __forceinline__ uint32_t topk_shift(int32_t lo, int32_t hi)
{
    uint32_t sh = 0;
    while (((int64_t(hi) - lo) >> sh) >= kSelBins) ++sh;
    return sh;
}

__device__ __forceinline__ int topk_bin(uint64_t key, int32_t lo, uint32_t sh)
{
    return int((int64_t(key_score(key)) - lo) >> sh);
}

// From the bin counts in s.hist: s.hist2[b] = start of bin b's segment (a
// segment ends where the next lower bin's starts), s.hist[b] = the same start
// (a write cursor for the scatter), and the cut. All threads get the result.
template <int BLOCK>
__device__ TopkCut topk_cut_from_hist(int64_t n, int k, int32_t lo, uint32_t sh, SelectSmem& s)
{
    __shared__ int32_t c_cut, c_above, c_tcount, c_maxseg;
    const int tid = threadIdx.x;
    if (tid == 0) {
        c_cut = -1;
        c_above = int32_t(n < k ? n : k);
        c_tcount = 0;
        c_maxseg = 0;
    }
    constexpr int PER = kSelBins / BLOCK > 0 ? kSelBins / BLOCK : 1;
    const int owners = kSelBins / PER;
    uint32_t local = 0;
    if (tid < owners)
        for (int j = 0; j < PER; ++j) local += s.hist[kSelBins - 1 - (tid * PER + j)];
    uint32_t total;
    uint32_t run = block_excl_scan<BLOCK>(local, s.part, total);
    int mseg = 0;
    if (tid < owners)
        for (int j = 0; j < PER; ++j) {
            const int bin = kSelBins - 1 - (tid * PER + j);
            const uint32_t c = s.hist[bin];
            s.hist2[bin] = run;
            s.hist[bin] = run;
            if (n > k && run < uint32_t(k) && uint32_t(k) <= run + c) {
                c_cut = bin;
                c_above = int32_t(run);
                c_tcount = int32_t(c);
            }
            if (run + c <= uint32_t(k) && int(c) > mseg) mseg = int(c);
            run += c;
        }
    if (mseg > 0) atomicMax(&c_maxseg, mseg);
    __syncthreads();
    TopkCut t;
    t.lo = lo;
    t.sh = sh;
    t.cut = c_cut;
    t.above = c_above;
    t.tcount = c_tcount;
    t.m = n < k ? int(n) : k;
    t.maxseg = c_maxseg;
    __syncthreads();  // the shared fields may be rewritten by a later call
    return t;
}

// Choose the cut bin's best (m - above) keys into tmp[above, m). `tie` holds
// the cut bin's tcount keys (shared or global; nullptr when they were not
// kept); without them the threshold is selected over all n `keys`.
template <int BLOCK>
__device__ void topk_take_ties(const TopkCut& t, const uint64_t* tie, const uint64_t* keys, int64_t n, uint64_t* tmp,
                               SelectSmem& s, uint32_t* err)
{
    __shared__ int32_t r_pos;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int need = t.m - t.above;
    if (need <= 0) return;
    if (tie != nullptr && t.tcount <= 64) {
        // one warp: a tie key's rank among the tie keys is its place
        if (warp == 0) {
            const uint64_t k1 = lane < t.tcount ? tie[lane] : 0ull;
            const uint64_t k2 = lane + 32 < t.tcount ? tie[lane + 32] : 0ull;
            int r1 = 0, r2 = 0;
            for (int j = 0; j < 32; ++j) {
                const uint64_t o1 = __shfl_sync(0xffffffffu, k1, j), o2 = __shfl_sync(0xffffffffu, k2, j);
                r1 += int(o1 > k1) + int(o2 > k1);
                r2 += int(o1 > k2) + int(o2 > k2);
            }
            if (k1 != 0ull && r1 < need) tmp[t.above + r1] = k1;
            if (k2 != 0ull && r2 < need) tmp[t.above + r2] = k2;
        }
        __syncthreads();
        return;
    }
    const uint64_t* src = tie != nullptr ? tie : keys;
    const int64_t ns = tie != nullptr ? int64_t(t.tcount) : n;
    const int64_t want = tie != nullptr ? int64_t(need) : int64_t(t.m);
    uint64_t thr = 1;
    if (want < ns) thr = block_select_threshold<BLOCK>(src, ns, want, s, err);
    if (tid == 0) r_pos = 0;
    __syncthreads();
    for (int64_t i = tid; i < ns; i += BLOCK) {
        const uint64_t key = src[i];
        if (key >= thr && key != 0ull && topk_bin(key, t.lo, t.sh) == t.cut) {
            const int pos = atomicAdd(&r_pos, 1);
            if (pos < need) tmp[t.above + pos] = key;
        }
    }
    __syncthreads();
    if (tid == 0 && r_pos != need) set_error(err, kErrSelectCount);
    __syncthreads();
}

// Order tmp[0, m) (bins above the cut in their segments, then the cut bin's
// keys) into out[0, m), descending. s.hist2 holds the segment starts. A key's
// place is its rank in its segment (one pass over the segment per key), up to
// kRankSegMax keys per segment; longer segments (many equal or close scores)
// sort everything with the bitonic network instead.
constexpr int kRankSegMax = 256;
template <int BLOCK>
__device__ void topk_rank(const TopkCut& t, const uint64_t* tmp, uint64_t* out, SelectSmem& s)
{
    const int tid = threadIdx.x;
    const int m = t.m, above = t.above;
    if (t.maxseg > kRankSegMax || m - above > kRankSegMax) {
        for (int i = tid; i < m; i += BLOCK) out[i] = tmp[i];
        __syncthreads();
        block_bitonic_desc<BLOCK>(out, m);
        return;
    }
    for (int p = tid; p < m; p += BLOCK) {
        const uint64_t key = tmp[p];
        int beg, end;
        if (p >= above) {
            beg = above;
            end = m;
        } else {
            const int b = topk_bin(key, t.lo, t.sh);  // b > cut >= -1
            beg = int(s.hist2[b]);
            end = b > 0 ? int(s.hist2[b - 1]) : m;
        }
        int r = 0;
        for (int j = beg; j < end; ++j) r += tmp[j] > key ? 1 : 0;
        out[beg + r] = key;
    }
    __syncthreads();
}

// Top-k of n unique keys, sorted descending (score desc, then id asc), in one
// CTA: range (unless `range_known`, when [lo, hi] must contain every score),
// histogram, cut, one scatter pass, ties, ranks. Writes min(n, k) keys to
// out[] and returns that count. `keys` may be shared or global memory (each
// pass keeps eight loads per thread in flight). out[] needs next_pow2(k) keys,
// tmp[] k keys, tie[] tie_cap keys.
template <int BLOCK>
__device__ int block_topk_sorted(const uint64_t* keys, int64_t n, int k, uint64_t* out, uint64_t* tmp,
                                 uint64_t* tie, int tie_cap, bool range_known, int32_t lo, int32_t hi,
                                 SelectSmem& s, uint32_t* err)
{
    constexpr int NW = BLOCK / 32;
    constexpr int U = 8;  // loads in flight per thread and pass
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ int32_t t_lo, t_tpos;
    __shared__ uint32_t t_sh;
    if (n <= 0) {
        __syncthreads();
        return 0;
    }
    auto for_keys = [&](auto&& fn) {
        for (int64_t base = 0; base < n; base += int64_t(BLOCK) * U) {
            uint64_t v[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t i = base + int64_t(u) * BLOCK + tid;
                v[u] = i < n ? keys[i] : 0ull;
            }
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (base + int64_t(u) * BLOCK + tid < n) fn(v[u]);
        }
    };
    if (!range_known) {
        lo = INT32_MAX;
        hi = INT32_MIN;
        for_keys([&](uint64_t key) {
            const int32_t sc = key_score(key);
            lo = sc < lo ? sc : lo;
            hi = sc > hi ? sc : hi;
        });
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, off));
            hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, off));
        }
        if (lane == 0) {
            s.red_lo[warp] = (unsigned long long)(uint32_t(lo));
            s.red_hi[warp] = (unsigned long long)(uint32_t(hi));
        }
    }
    for (int i = tid; i < kSelBins; i += BLOCK) s.hist[i] = 0;
    __syncthreads();
    if (tid == 0) {
        int32_t l = lo, h = hi;
        if (!range_known) {
            l = INT32_MAX;
            h = INT32_MIN;
            for (int w = 0; w < NW; ++w) {
                l = min(l, int32_t(uint32_t(s.red_lo[w])));
                h = max(h, int32_t(uint32_t(s.red_hi[w])));
            }
        }
        t_lo = l;
        t_sh = topk_shift(l, h);
        t_tpos = 0;
    }
    __syncthreads();
    const int32_t base = t_lo;
    const uint32_t sh = t_sh;
    for_keys([&](uint64_t key) { atomicAdd(&s.hist[topk_bin(key, base, sh)], 1u); });
    __syncthreads();
    const TopkCut t = topk_cut_from_hist<BLOCK>(n, k, base, sh, s);
    const bool tie_fits = t.tcount <= tie_cap;
    // scatter the bins above the cut to their segments; gather the cut bin
    for_keys([&](uint64_t key) {
        const int b = topk_bin(key, base, sh);
        if (b > t.cut) {
            tmp[atomicAdd(&s.hist[b], 1u)] = key;
        } else if (b == t.cut && tie_fits) {
            tie[atomicAdd(&t_tpos, 1)] = key;
        }
    });
    __syncthreads();
    topk_take_ties<BLOCK>(t, tie_fits ? tie : nullptr, keys, n, tmp, s, err);
    topk_rank<BLOCK>(t, tmp, out, s);
    return t.m;
}

__host__ __device__ __forceinline__ int next_pow2(int v)
{
    int p = 1;
    while (p < v) p <<= 1;
    return p;
}

// Raise a kernel's dynamic shared memory limit to at least `bytes`, once per
// device and kernel.
cudaError_t ensure_smem_attr(const void* func, int bytes);

// ----------------------------------------------------------------------------
// Kernel launchers (defined in the .cu files)
// ----------------------------------------------------------------------------
int probe_slices(const SearchArgs& a, int num_sms);
cudaError_t launch_probe_search(const SearchArgs& a, int num_sms, cudaStream_t s);
size_t probe_noalloc_scratch_bytes(int B, int S, int P, int nlist, bool keys_in_smem);
cudaError_t launch_probe_noalloc(SearchArgs a, int S, cudaStream_t s);
cudaError_t launch_plan(const SearchArgs& a, int num_sms, cudaStream_t s);

cudaError_t launch_scan(const SearchArgs& a, int num_sms, cudaStream_t s);
// tmaps: the index's item rows as two 2-D tensor maps (opaque CUtensorMap, 128
// bytes each): tiles of 32 rows, then of 128 rows
cudaError_t launch_scan_tc(const SearchArgs& a, const void* tmaps, int num_sms, cudaStream_t s);
bool scan_tc_supported(int d);
cudaError_t launch_select(const SearchArgs& a, int num_sms, cudaStream_t s);
bool select_reads_bins(int B, int k);  // the final top-k reads the scans' score bins
cudaError_t launch_merge(const int64_t* ids, const int32_t* scores, int G, int B, int k, int64_t* out_ids,
                         int32_t* out_scores, cudaStream_t s);
cudaError_t merge_error_word(uint32_t* word, bool clear);
size_t scan_smem_bytes(int d, int W);
// Where the rows of an index live, for the update, insert and delete kernels:
// rows [0, n) are the creation lists (list c: offsets[c] .. offsets[c+1]-1, plane
// blocks from base_chunk_start[c]); rows n + kWarpItems * a + r (r < app_len[a])
// are append chunk a, plane block n_base_chunks + a.
struct RowMap {
    const int64_t* offsets;
    const int32_t* base_chunk_start;
    int32_t nlist;
    int64_t n;
    int32_t n_base_chunks;
    const int32_t* app_len;  // [n_app] rows filled in each append chunk
    int32_t n_app;
};
cudaError_t launch_delete(uint32_t* dead, const RowMap& map, const int64_t* ids, int64_t m, uint32_t* err,
                          cudaStream_t s);
cudaError_t launch_update(int8_t* items, uint64_t* sigs, uint32_t* planes, const RowMap& map, int d, int W,
                          const int64_t* ids, const int8_t* new_items, const uint64_t* new_sigs, int64_t m,
                          uint32_t* err, cudaStream_t s);
cudaError_t launch_build_planes(const uint64_t* sigs, const int64_t* offsets, const int32_t* chunk_start,
                                const int32_t* chunk_list, int32_t n_chunks, int W, uint32_t* planes,
                                cudaStream_t s);

}  // namespace st
