// Internal definitions shared by the libst kernels and the host API.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/st.h"

namespace st {

// ----------------------------------------------------------------------------
// Tunables of the list scan
// ----------------------------------------------------------------------------
constexpr int kScanBlock = 128;            // threads per scan CTA (independent warps)
constexpr int kWarpItems = 256;            // list rows per work unit (one warp)
constexpr int kQMax = 32;                  // queries per work unit (one bit each)
constexpr int kExpandBlock = 256;

constexpr int kProbeBlock = 512;
constexpr int kProbeSmemKeys = 16384;      // nlist up to this keeps probe keys in smem
constexpr int kSelectBlock = 1024;
constexpr int kSelectSmemKeys = 16384;     // candidates up to this are selected in smem
constexpr int kPlanBlock = 1024;

// Device error word bits (st_index_check reports any of them as ST_ERR_DEVICE).
enum : uint32_t {
    kErrUnitDecode = 1u << 0,   // a work unit index did not map to a list
    kErrQueryGroup = 1u << 1,   // a query group exceeded kQMax
    kErrSelectCount = 1u << 2,  // a selection collected the wrong number of keys
    kErrOverflowPath = 1u << 3, // the exact overflow path met an impossible state
    kErrUnitTable = 1u << 4,    // more work units than the host-sized table holds
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
// Per-search plan written by the plan kernel and read by the scan kernel.
// ----------------------------------------------------------------------------
struct PlanCtl {
    int32_t n_units;       // work units of this search
    int32_t n_lists;       // distinct probed lists
    int32_t next_unit;     // dynamic work counter of the scan kernel
    int32_t pad;
};

struct SearchArgs {
    // index (read-only)
    const int8_t* items;
    const uint64_t* sigs;
    const int64_t* offsets;
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
    // scratch
    int32_t* probe;          // [B][P]
    uint64_t* probe_keys;    // [B][nlist] when nlist > kProbeSmemKeys, else null
    int32_t* list_cnt;       // [nlist] queries probing each list
    int32_t* list_qstart;    // [nlist]
    int32_t* list_fill;      // [nlist]
    int32_t* qlist;          // [B*P] query ids grouped by list
    int32_t* dl_list;        // [min(nlist, B*P)] distinct probed lists
    int32_t* dl_qstart;      // [..]
    int32_t* dl_qcnt;        // [..]
    int32_t* dl_ustart;      // [.. + 1] first unit of each distinct list
    int4* units;             // [max_units] {first row, rows, qlist offset, queries}
    int32_t max_units;
    PlanCtl* ctl;
    uint32_t* cand_cnt;      // [B] candidates emitted per query (may exceed cap)
    uint64_t* cand;          // [B][cap]
    int64_t cap;             // candidate keys per query
    unsigned long long* eligible_cnt;  // [B]
    uint32_t* err;           // device error word
};

// ----------------------------------------------------------------------------
// int8 inner products with dp4a (4 signed byte products added into int32)
// ----------------------------------------------------------------------------
__device__ __forceinline__ int32_t dot16(const int4 a, const int4 b, int32_t acc)
{
    acc = __dp4a(a.x, b.x, acc);
    acc = __dp4a(a.y, b.y, acc);
    acc = __dp4a(a.z, b.z, acc);
    acc = __dp4a(a.w, b.w, acc);
    return acc;
}

__device__ __forceinline__ void set_error(uint32_t* err, uint32_t bit)
{
    atomicOr(err, bit);
}

__device__ __forceinline__ unsigned lanemask_lt()
{
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// ----------------------------------------------------------------------------
// Block-wide selection primitives (one CTA, BLOCK threads).
// ----------------------------------------------------------------------------
struct SelectSmem {
    uint32_t hist[256];
    uint64_t prefix;
    int64_t krem;
    int32_t count;
};

// The k-th largest of n unique keys (1 <= k <= n), by MSB-first radix select
// with 8-bit digits. `keys` may be shared or global memory.
template <int BLOCK>
__device__ uint64_t block_kth_largest(const uint64_t* keys, int64_t n, int64_t k, SelectSmem& s)
{
    if (threadIdx.x == 0) {
        s.prefix = 0;
        s.krem = k;
    }
    __syncthreads();
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += BLOCK) s.hist[i] = 0;
        __syncthreads();
        const uint64_t prefix = s.prefix;
        for (int64_t i = threadIdx.x; i < n; i += BLOCK) {
            const uint64_t key = keys[i];
            const bool match = (shift == 56) || ((key >> (shift + 8)) == prefix);
            if (match) atomicAdd(&s.hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            const int lane = threadIdx.x;
            // lane owns bins [8*lane, 8*lane+8); walk from the top bin down
            uint32_t c[8];
            uint32_t sum = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                c[j] = s.hist[8 * lane + j];
                sum += c[j];
            }
            // exclusive suffix sum over lanes above this one
            uint32_t incl = sum;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const uint32_t v = __shfl_down_sync(0xffffffffu, incl, off);
                if (lane + off < 32) incl += v;
            }
            const int64_t above = int64_t(incl - sum);
            const int64_t krem = s.krem;
            if (above < krem && krem <= above + int64_t(sum)) {
                int64_t acc = above;
                for (int j = 7; j >= 0; --j) {
                    if (acc + c[j] >= krem) {
                        s.prefix = (prefix << 8) | uint64_t(8 * lane + j);
                        s.krem = krem - acc;
                        break;
                    }
                    acc += c[j];
                }
            }
        }
        __syncthreads();
    }
    return s.prefix;
}

// Copy every key >= kth from keys[0..n) into out[]; returns the count.
template <int BLOCK>
__device__ int32_t block_collect_ge(const uint64_t* keys, int64_t n, uint64_t kth, uint64_t* out,
                                    int32_t out_cap, SelectSmem& s)
{
    if (threadIdx.x == 0) s.count = 0;
    __syncthreads();
    for (int64_t i = threadIdx.x; i < n; i += BLOCK) {
        const uint64_t key = keys[i];
        if (key >= kth) {
            const int32_t pos = atomicAdd(&s.count, 1);
            if (pos < out_cap) out[pos] = key;
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

// Raise a kernel's dynamic shared memory limit to 200 KiB, once per device and
// kernel slot (slot < 16). Setting it twice is harmless, so a race only repeats it.
cudaError_t ensure_smem_attr(const void* func, int slot);

// ----------------------------------------------------------------------------
// Kernel launchers (defined in the .cu files)
// ----------------------------------------------------------------------------
cudaError_t launch_probe(const SearchArgs& a, cudaStream_t s);
cudaError_t launch_plan(const SearchArgs& a, int num_sms, cudaStream_t s);
cudaError_t launch_scan(const SearchArgs& a, int num_sms, cudaStream_t s);
cudaError_t launch_select(const SearchArgs& a, cudaStream_t s);

}  // namespace st
