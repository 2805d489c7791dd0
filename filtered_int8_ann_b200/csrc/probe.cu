// Coarse probe: score every IVF centroid against each query with int32
// accumulation and keep the query's nprobe best lists, best first (score
// descending, lower list id first among equal scores).
//
// "Pick the most promising clusters first, filter only inside them, then score
// only the survivors" -- SilverTorch: Index as Model, section on how each
// component worked before. The pages name probes (64 of them with top-2048)
// but not the index type; this library reads it as an IVF with int8 centroids
// and contiguous lists.
//
// Grid: B queries x S centroid slices (S chosen so the grid fills the GPU).
// Each CTA scores its slice (16-byte read-only loads of centroid rows from L2,
// dp4a against the query held in shared memory, unrolled for memory-level
// parallelism), keeps its slice's nprobe best keys (exact: the global top-P is
// a subset of the union of the slices' top-P) and publishes them. The last CTA
// of a query to finish -- found with one atomic counter, no waiting -- merges
// the S partial lists, writes the probe result, and files the query into every
// chosen list: it takes the next rank of the list's query counter and writes
// its id and mask into the list's slot row, which the plan and the scan read.
#include <mutex>

#include "st_internal.cuh"

namespace st {

// kFile: also file the query into its lists (the search); the allocation-free
// probe-only call sets it false and writes the probe result alone.
template <int BLOCK, bool kFile>
__device__ void finish_query(const SearchArgs& a, int b, uint64_t* keys, int n, uint64_t* sortbuf,
                             int pw, SelectSmem& ss)
{
    const int P = a.P;
    uint64_t thr = 1;  // key 0 marks an empty partial slot and is never a real key
    if (P < n) thr = block_select_threshold<BLOCK>(keys, n, P, ss, a.err);
    const int got = block_collect_ge<BLOCK>(keys, n, thr < 1 ? 1 : thr, sortbuf, pw, ss);
    if (threadIdx.x == 0 && got != P) set_error(a.err, kErrSelectCount);
    for (int i = (got < pw ? got : pw) + threadIdx.x; i < pw; i += BLOCK) sortbuf[i] = 0;
    __syncthreads();
    block_sort_desc_counting<BLOCK>(sortbuf, got < pw ? got : pw, keys, ss);  // the score keys are done with
    if (!kFile) {
        for (int p = threadIdx.x; p < P; p += BLOCK) a.probe[int64_t(b) * P + p] = int(key_id(sortbuf[p]));
        return;
    }
    const int W = a.W;
    // the query's mask bits in increasing order
    if (threadIdx.x < 32) {
        const uint64_t m0 = a.qmasks[int64_t(b) * W];
        const uint64_t m1 = W > 1 ? a.qmasks[int64_t(b) * W + 1] : 0ull;
        const int lane = threadIdx.x;
        int n_before = 0;
        for (int r = 0; r < 2 * W; ++r) {
            const int bit = 32 * r + lane;
            const uint64_t word = bit < 64 ? m0 : m1;
            const bool on = (word >> (bit & 63)) & 1ull;
            const unsigned bal = __ballot_sync(0xffffffffu, on);
            if (on) a.qbits[int64_t(b) * kMaskBitsMax + n_before + __popc(bal & lanemask_lt())] = uint8_t(bit);
            n_before += __popc(bal);
        }
        if (lane == 0) a.qnbits[b] = n_before;
    }
    for (int p = threadIdx.x; p < P; p += BLOCK) {
        const int L = int(key_id(sortbuf[p]));
        a.probe[int64_t(b) * P + p] = L;
        if (L >= 0 && L < a.nlist) {
            const int r = atomicAdd(&a.list_cnt[L], 1);
            const int64_t slot = int64_t(L) * a.B + r;
            a.qlist[slot] = b;
            const uint64_t m0 = a.qmasks[int64_t(b) * W];
            const uint64_t m1 = W > 1 ? a.qmasks[int64_t(b) * W + 1] : 0ull;
            reinterpret_cast<ulonglong2*>(a.qmask_slot)[slot] = make_ulonglong2(m0, m1);
        }
    }
}

template <int BLOCK, bool kFile>
__global__ void __launch_bounds__(BLOCK)
probe_kernel(SearchArgs a, int S)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ SelectSmem ss;
    __shared__ int s_last;
    const int b = blockIdx.x / S;
    const int sl = blockIdx.x - b * S;
    const int d = a.d;
    const int nlist = a.nlist;
    const int P = a.P;
    const int pw = next_pow2(P);
    const int pws = pw > BLOCK ? pw : BLOCK;  // the sort pads to at least BLOCK keys
    const int c0 = int(int64_t(sl) * nlist / S), c1 = int(int64_t(sl + 1) * nlist / S);
    const int nloc = c1 - c0;

    // shared layout: [sort buffer pws keys][query d bytes][keys of the slice (if local)]
    uint64_t* sortbuf = reinterpret_cast<uint64_t*>(smem_raw);
    int4* qv = reinterpret_cast<int4*>(sortbuf + pws);
    const bool local_keys = (a.probe_keys == nullptr);
    uint64_t* keys = local_keys ? reinterpret_cast<uint64_t*>(qv + d / 16)
                                : a.probe_keys + int64_t(b) * nlist + c0;

    const int4* q4 = reinterpret_cast<const int4*>(a.queries + int64_t(b) * d);
    for (int j = threadIdx.x; j < d / 16; j += BLOCK) qv[j] = q4[j];
    __syncthreads();

    const int np = d / 16;
    constexpr int U = 4;  // centroid rows per thread in flight
    for (int cb = threadIdx.x; cb < nloc; cb += BLOCK * U) {
        int32_t acc[U];
#pragma unroll
        for (int u = 0; u < U; ++u) acc[u] = 0;
        for (int p = 0; p < np; ++p) {
            const int4 qp = qv[p];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = cb + u * BLOCK;
                if (c < nloc)
                    acc[u] = dot16(__ldg(reinterpret_cast<const int4*>(a.centroids + int64_t(c0 + c) * d) + p),
                                   qp, acc[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = cb + u * BLOCK;
            if (c < nloc) keys[c] = pack_key(acc[u], uint32_t(c0 + c));
        }
    }
    __syncthreads();

    if (S == 1) {
        finish_query<BLOCK, kFile>(a, b, keys, nloc, sortbuf, pw, ss);
        return;
    }

    // this slice's best min(P, nloc) keys -> its partial row (zeros fill the rest)
    const int Pl = P < nloc ? P : nloc;
    uint64_t thr = 0;
    if (Pl < nloc) thr = block_select_threshold<BLOCK>(keys, nloc, Pl, ss, a.err);
    uint64_t* part = a.probe_part + (int64_t(b) * S + sl) * P;
    const int got = block_collect_ge<BLOCK>(keys, nloc, thr, sortbuf, pw, ss);
    if (threadIdx.x == 0 && got != Pl) set_error(a.err, kErrSelectCount);
    for (int i = threadIdx.x; i < P; i += BLOCK) part[i] = i < got ? sortbuf[i] : 0ull;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(&a.probe_done[b], 1) == S - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    // last slice of this query: merge the S partial rows (S*S*P <= nlist, so
    // S*P keys fit the slice key space, local or global)
    const int n = S * P;
    uint64_t* mk = local_keys ? keys : a.probe_keys + int64_t(b) * nlist;
    const uint64_t* src = a.probe_part + int64_t(b) * S * P;
    for (int i = threadIdx.x; i < n; i += BLOCK) mk[i] = __ldcg(src + i);
    __syncthreads();
    finish_query<BLOCK, kFile>(a, b, mk, n, sortbuf, pw, ss);
}

int probe_slices(const SearchArgs& a, int num_sms)
{
    // enough CTAs to cover the GPU twice, slices of at least 1024 centroids,
    // and the merged partial rows (S * nprobe keys) must fit the key space
    int S = (2 * num_sms + a.B - 1) / a.B;
    const int by_size = a.nlist / 1024;
    if (S > by_size) S = by_size;
    if (S > 32) S = 32;
    while (S > 1 && int64_t(S) * S * a.P > a.nlist) --S;  // merged rows fit one slice's key space
    if (S < 1) S = 1;
    return S;
}

static size_t probe_smem_bytes(const SearchArgs& a, int S)
{
    const int pw = next_pow2(a.P);
    size_t bytes = size_t(pw > kProbeBlock ? pw : kProbeBlock) * 8 + size_t(a.d);
    if (a.probe_keys == nullptr) bytes += size_t((a.nlist + S - 1) / S + 1) * 8;
    return bytes;
}

cudaError_t launch_probe(const SearchArgs& a, int S, cudaStream_t s)
{
    const size_t smem = probe_smem_bytes(a, S);
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(probe_kernel<kProbeBlock, true>), 0, 200 * 1024);
    if (e != cudaSuccess) return e;
    probe_kernel<kProbeBlock, true><<<a.B * S, kProbeBlock, smem, s>>>(a, S);
    return cudaGetLastError();
}

// ----------------------------------------------------------------------------
// Allocation-free probe (st_probe_noalloc). Its scratch -- the per-query
// completion counters, the slices' partial top-P rows and, for very large
// nlist, the centroid score keys -- lives in this fixed device array instead
// of memory allocated per call. Every call uses the same array.
// ----------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_probe_scratch[ST_PROBE_NOALLOC_SCRATCH_BYTES];

size_t probe_noalloc_scratch_bytes(int B, int S, int P, int nlist, bool keys_in_smem)
{
    size_t bytes = (size_t(B) * 4 + 255) / 256 * 256;  // completion counters
    bytes += size_t(B) * S * P * 8;                       // partial rows
    if (!keys_in_smem) bytes += size_t(B) * nlist * 8;    // score keys
    return bytes;
}

cudaError_t launch_probe_noalloc(SearchArgs a, int S, cudaStream_t s)
{
    // device address of the array, looked up once per device
    static std::mutex mu;
    static unsigned char* base_of[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64) return cudaErrorInvalidDevice;
    unsigned char* base = nullptr;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (base_of[dev] == nullptr) {
            void* ptr = nullptr;
            e = cudaGetSymbolAddress(&ptr, g_probe_scratch);
            if (e != cudaSuccess) return e;
            base_of[dev] = static_cast<unsigned char*>(ptr);
        }
        base = base_of[dev];
    }
    const size_t done_bytes = (size_t(a.B) * 4 + 255) / 256 * 256;
    a.probe_done = reinterpret_cast<int32_t*>(base);
    a.probe_part = reinterpret_cast<uint64_t*>(base + done_bytes);
    if (a.probe_keys != nullptr)  // non-null marks "keys in global memory"
        a.probe_keys = reinterpret_cast<uint64_t*>(base + done_bytes + size_t(a.B) * S * a.P * 8);
    e = cudaMemsetAsync(a.probe_done, 0, size_t(a.B) * 4, s);
    if (e != cudaSuccess) return e;
    const size_t smem = probe_smem_bytes(a, S);
    e = ensure_smem_attr(reinterpret_cast<const void*>(probe_kernel<kProbeBlock, false>), 9, 200 * 1024);
    if (e != cudaSuccess) return e;
    probe_kernel<kProbeBlock, false><<<a.B * S, kProbeBlock, smem, s>>>(a, S);
    return cudaGetLastError();
}

}  // namespace st
