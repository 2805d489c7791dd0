// Internal definitions shared by the libst kernels and the host API.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/st.h"

namespace st {

// ----------------------------------------------------------------------------
// Tunables
// ----------------------------------------------------------------------------
constexpr int kScanBlock = 32;             // threads per scan CTA (one independent warp)
constexpr int kWarpItems = 512;            // list rows per work unit (one warp)
constexpr int kQMax = 32;                  // queries per work unit (one bit each)

constexpr int kProbeBlock = 512;
constexpr int kProbeSmemKeys = 16384;      // nlist up to this keeps probe keys in smem
constexpr int kSelectBlock = 1024;
constexpr int kSelectSmemKeys = 22528;     // candidates up to this are selected in smem
constexpr int kPlanBlock = 512;
constexpr int kSelBits = 11;               // radix digit of the selections
constexpr int kSelBins = 1 << kSelBits;
constexpr uint32_t kWaitLimit = 1u << 24;  // bounded mbarrier polls before giving up

// Device error word bits (st_index_check reports any of them as ST_ERR_DEVICE).
enum : uint32_t {
    kErrUnitDecode = 1u << 0,   // a work unit did not map to a list
    kErrQueryGroup = 1u << 1,   // a query group exceeded kQMax
    kErrSelectCount = 1u << 2,  // a selection collected the wrong number of keys
    kErrOverflowPath = 1u << 3, // the exact overflow path met an impossible state
    kErrUnitTable = 1u << 4,    // more work units than the host-sized table holds
    kErrCopyTimeout = 1u << 5,  // a bulk copy did not complete within the wait bound
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
    int32_t n_units;       // work units of this search
    int32_t pad[3];
};

struct SearchArgs {
    // index (read-only)
    const int8_t* items;
    const uint64_t* sigs;
    const int64_t* offsets;
    const int32_t* nchunks;  // [nlist] ceil(list rows / kWarpItems)
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
    // scratch (the zeroed block first: one memset clears it)
    int32_t* list_cnt;       // [nlist] queries probing each list        (zeroed)
    int32_t* list_fill;      // [nlist] scatter cursor                    (zeroed)
    uint32_t* cand_cnt;      // [B] candidates reserved per query         (zeroed)
    unsigned long long* eligible_cnt;  // [B]                             (zeroed)
    PlanCtl* ctl;            //                                           (zeroed)
    int32_t* probe;          // [B][P]
    uint64_t* probe_keys;    // [B][nlist] when nlist > kProbeSmemKeys, else null
    int32_t* list_qstart;    // [nlist] first query slot of each list
    int32_t* qlist;          // [B*P] query id of each slot (slots grouped by list)
    uint64_t* qmask_slot;    // [B*P][2] that query's mask words (word 1 = 0 when W = 1)
    int4* units;             // [max_units] {first row, rows, first slot, queries}
    int32_t max_units;
    uint64_t* cand;          // [B][cap]
    int64_t cap;             // candidate keys per query
    uint32_t* err;           // device error word
};

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

// mbarrier + bulk async copy (global -> this CTA's shared memory; never multicast)
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Poll the barrier phase at most kWaitLimit times; false if it never completed.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity)
{
    for (uint32_t it = 0; it < kWaitLimit; ++it)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// Order this thread's generic-proxy shared-memory accesses before later
// async-proxy (bulk copy) accesses to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 16-byte asynchronous copy global -> shared (cp.async, L1-allocating)
__device__ __forceinline__ void cp_async16(void* dst, const void* src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// ----------------------------------------------------------------------------
// Block-wide selection (one CTA of BLOCK threads)
// ----------------------------------------------------------------------------
struct SelectSmem {
    uint32_t hist[kSelBins];
    uint32_t part[32];
    unsigned long long red_lo[32], red_hi[32];
    uint64_t prefix;     // high bits of the threshold fixed so far
    int64_t krem;        // rank still to find below the prefix
    int32_t shift;       // bits below the prefix
    int32_t done;
    int32_t found;
    int32_t count;
};

// Warp-aggregated shared histogram increment. Every lane of the warp calls it.
__device__ __forceinline__ void hist_add(uint32_t* hist, bool active, uint32_t bin)
{
    const unsigned act = __ballot_sync(0xffffffffu, active);
    if (!active) return;
    const unsigned peers = __match_any_sync(act, bin);
    if (int(threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], uint32_t(__popc(peers)));
}

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
// score's high bits are shared by all candidates), 11-bit digits, warp-
// aggregated histogram updates, and an early exit as soon as the bucket holding
// the k-th key is taken whole. `keys` may be shared or global memory.
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
        for (int64_t base = 0; base < n; base += BLOCK) {
            const int64_t i = base + tid;
            bool act = false;
            uint32_t bin = 0;
            if (i < n) {
                const uint64_t x = keys[i];
                act = shift_hi >= 64 || (x >> shift_hi) == (prefix >> shift_hi);
                bin = uint32_t(x >> shift) & uint32_t(nb - 1);
            }
            hist_add(s.hist, act, bin);
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
    return s.count;
}

// Sort m keys (m a power of two) in shared memory, descending.
template <int BLOCK>
__device__ void block_bitonic_desc(uint64_t* a, int m)
{
    for (int size = 2; size <= m; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = threadIdx.x; i < (m >> 1); i += BLOCK) {
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

__host__ __device__ __forceinline__ int next_pow2(int v)
{
    int p = 1;
    while (p < v) p <<= 1;
    return p;
}

// Raise a kernel's dynamic shared memory limit, once per device and kernel slot
// (slot < 32). Setting it twice is harmless, so a race only repeats it.
cudaError_t ensure_smem_attr(const void* func, int slot, int bytes);

// ----------------------------------------------------------------------------
// Kernel launchers (defined in the .cu files)
// ----------------------------------------------------------------------------
cudaError_t launch_probe(const SearchArgs& a, cudaStream_t s);
cudaError_t launch_plan(const SearchArgs& a, int num_sms, cudaStream_t s);
cudaError_t launch_scan(const SearchArgs& a, int num_sms, cudaStream_t s);
cudaError_t launch_select(const SearchArgs& a, cudaStream_t s);
size_t scan_smem_bytes(int d, int W);

}  // namespace st
