// Exact merge of document-shard top-k lists: for each query, the k best keys
// (score descending, then id ascending) of the union of the shards' lists.
// With disjoint shards every item of the global top-k is in its own shard's
// top-k, so the merge reproduces the unsharded search. Document sharding is how
// the pages scale out once one GPU is used up (SilverTorch: Index as Model,
// section on engineering for scale and freshness, vertical and horizontal
// scaling paragraph).
//
// One CTA per query: the G*k (id, score) pairs become 64-bit keys in shared
// memory (padding entries, id -1, are dropped), and block_topk_sorted picks
// and orders the k best.
#include "st_internal.cuh"

namespace st {

// Device error word of the merge (per device: the kernel records an id out of
// range here; st_merge_check reads and clears it).
static __device__ uint32_t g_merge_err;

constexpr int kMergeBlock = 1024;
constexpr int kMergeTieCap = 1024;

// Is `key` in list g' (ordered like st_search: keys descending, padding last)?
__device__ __forceinline__ bool in_sorted_list(const int64_t* ids, const int32_t* scores, int64_t row, int k,
                                               uint64_t key)
{
    int lo = 0, hi = k - 1;  // the first position whose key is <= `key`
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        const int64_t id = ids[row + mid];
        const uint64_t km = id >= 0 ? pack_key(scores[row + mid], uint32_t(id)) : 0ull;
        if (km > key) lo = mid + 1;
        else hi = mid;
    }
    const int64_t id = ids[row + lo];
    return id >= 0 && pack_key(scores[row + lo], uint32_t(id)) == key;
}

// UNION: drop a key that an earlier list already holds (one binary search per
// earlier list), so an item found by several lists is merged once.
template <bool UNION>
__global__ void __launch_bounds__(kMergeBlock)
merge_kernel(const int64_t* ids, const int32_t* scores, int G, int B, int k, int64_t* out_ids,
             int32_t* out_scores)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ SelectSmem ss;
    __shared__ int s_n;
    const int b = blockIdx.x;
    // shared layout: [tmp k keys, rounded up to even][tie kMergeTieCap keys]
    // [keys max(G*k, next_pow2(k)), reused as the output]
    uint64_t* tmp = reinterpret_cast<uint64_t*>(smem_raw);
    uint64_t* tie = tmp + ((k + 1) & ~1);
    uint64_t* keys = tie + kMergeTieCap;
    if (threadIdx.x == 0) s_n = 0;
    __syncthreads();
    const int total = G * k;
    for (int i0 = 0; i0 < total; i0 += kMergeBlock) {  // same trip count in every thread
        const int i = i0 + int(threadIdx.x);
        bool take = false;
        uint64_t key = 0;
        if (i < total) {
            const int g = i / k, r = i - g * k;
            const int64_t src = (int64_t(g) * B + b) * k + r;
            const int64_t id = ids[src];
            if (id >= 0 && id < (int64_t(1) << 31)) {
                key = pack_key(scores[src], uint32_t(id));
                take = true;
                if (UNION)
                    for (int h = 0; h < g && take; ++h)
                        take = !in_sorted_list(ids, scores, (int64_t(h) * B + b) * k, k, key);
            } else if (id != -1) {
                atomicOr(&g_merge_err, kErrUnitDecode);
            }
        }
        const unsigned bal = __ballot_sync(0xffffffffu, take);
        int base = 0;
        if ((threadIdx.x & 31) == 0 && bal) base = atomicAdd(&s_n, __popc(bal));
        base = __shfl_sync(0xffffffffu, base, 0);
        if (take) keys[base + __popc(bal & lanemask_lt())] = key;
    }
    __syncthreads();
    const int n = s_n;
    const int m = block_topk_sorted<kMergeBlock>(keys, n, k, keys, tmp, tie, kMergeTieCap, false, 0, 0, ss,
                                                 &g_merge_err);
    for (int r = threadIdx.x; r < k; r += kMergeBlock) {
        const uint64_t key = r < m ? keys[r] : 0ull;
        out_ids[int64_t(b) * k + r] = key == 0ull ? -1 : key_id(key);
        out_scores[int64_t(b) * k + r] = key_score(key);
    }
}

template <bool UNION>
static cudaError_t launch_merge_impl(const int64_t* ids, const int32_t* scores, int G, int B, int k,
                                     int64_t* out_ids, int32_t* out_scores, cudaStream_t s)
{
    const int pw = next_pow2(k);
    const int nkeys = G * k > pw ? G * k : pw;
    const size_t smem = (size_t((k + 1) & ~1) + kMergeTieCap + size_t(nkeys)) * 8;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(merge_kernel<UNION>),
                                     int((size_t(ST_SMALL_K) + kMergeTieCap + ST_MERGE_MAX_KEYS) * 8));
    if (e != cudaSuccess) return e;
    merge_kernel<UNION><<<B, kMergeBlock, smem, s>>>(ids, scores, G, B, k, out_ids, out_scores);
    return cudaGetLastError();
}

cudaError_t launch_merge(const int64_t* ids, const int32_t* scores, int G, int B, int k, int64_t* out_ids,
                         int32_t* out_scores, cudaStream_t s)
{
    return launch_merge_impl<false>(ids, scores, G, B, k, out_ids, out_scores, s);
}

cudaError_t launch_merge_union(const int64_t* ids, const int32_t* scores, int G, int B, int k, int64_t* out_ids,
                               int32_t* out_scores, cudaStream_t s)
{
    return launch_merge_impl<true>(ids, scores, G, B, k, out_ids, out_scores, s);
}

cudaError_t merge_error_word(uint32_t* word, bool clear)
{
    cudaError_t e = cudaMemcpyFromSymbol(word, g_merge_err, sizeof(uint32_t));
    if (e == cudaSuccess && clear && *word) {
        const uint32_t z = 0;
        e = cudaMemcpyToSymbol(g_merge_err, &z, sizeof(uint32_t));
    }
    return e;
}

}  // namespace st
