// Coarse probe: score every IVF centroid against each query with int32
// accumulation and keep the query's nprobe best lists, best first (score
// descending, lower list id first among equal scores).
//
// The most promising clusters are chosen first, the filter runs only inside
// them, and only the items that pass are scored -- SilverTorch: Index as Model,
// section on how each component worked before. The pages name probes (64 of them with top-2048)
// but not the index type; this library reads it as an IVF with int8 centroids
// and contiguous lists.
//
// The search runs the probe as two kernels:
//   * probe_score_kernel: one CTA per tile of 64 centroids x 64 queries; the
//     tile's queries sit in shared memory and every centroid row is read once
//     per tile (not once per query), dotted by dp4a against 16 queries per
//     thread, and the (score, list id) keys go to a [B][nlist] array that
//     stays in L2;
//   * probe_select_cluster_kernel: one thread-block cluster per query (up to
//     8 CTAs at small batches, so the whole GPU works on the selections). The
//     keys' a-priori score range [-128 sum|q_j|, 128 sum|q_j|], a 2048-bin
//     histogram over it summed through distributed shared memory, and the
//     suffix counts give the bin holding
//     the nprobe-th best score, so only the keys at or above that bin (a few
//     more than nprobe) reach the leader CTA for the exact selection and the
//     sort. The leader then writes the probe result and files the query into
//     every chosen list: it takes the next rank of the list's query counter
//     and writes its id and mask into the list's slot row, which the plan and
//     the scan read.
// The allocation-free probe-only call keeps an older single-kernel form (CTAs
// over query x centroid slices, last CTA merges), whose scratch is bounded.
#include <mutex>

#include "cluster_topk.cuh"

namespace st {

// Write the probe result of query b from its P best keys, sorted (sorted[p],
// p < P). kFile: also file the query into its lists (the search): the bits of
// each of its masks (its mask and its alternatives) in increasing order, then
// for each chosen list the next rank of the list's query counter and, in that
// slot of the list's slot row, the query's id, the union of its masks and the
// first kSlotBits bits of its mask. The allocation-free probe-only call writes the result alone.
template <int BLOCK, bool kFile>
__device__ void file_query(const SearchArgs& a, int b, const uint64_t* sorted)
{
    const int P = a.P;
    if (!kFile) {
        for (int p = threadIdx.x; p < P; p += BLOCK) a.probe[int64_t(b) * P + p] = int(key_id(sorted[p]));
        return;
    }
    const int W = a.W;
    const int n_alt = 1 + a.n_or;  // the query's masks: qmasks[b], then its alternatives
    __shared__ __align__(16) uint8_t s_bits[kSlotBits];
    __shared__ uint64_t s_union[2];
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        uint64_t u0 = 0, u1 = 0;
        for (int alt = 0; alt < n_alt; ++alt) {
            const uint64_t* mk = alt == 0 ? a.qmasks + int64_t(b) * W : a.or_masks + (int64_t(b) * a.n_or + alt - 1) * W;
            const uint64_t m0 = mk[0];
            const uint64_t m1 = W > 1 ? mk[1] : 0ull;
            u0 |= m0;
            u1 |= m1;
            const int64_t row = int64_t(b) * n_alt + alt;
            int n_before = 0;
            for (int r = 0; r < 2 * W; ++r) {
                const int bit = 32 * r + lane;
                const uint64_t word = bit < 64 ? m0 : m1;
                const bool on = (word >> (bit & 63)) & 1ull;
                const unsigned bal = __ballot_sync(0xffffffffu, on);
                const int j = n_before + __popc(bal & lanemask_lt());
                if (on) {
                    a.qbits[row * kMaskBitsMax + j] = uint8_t(bit);
                    if (alt == 0 && j < kSlotBits) s_bits[j] = uint8_t(bit);
                }
                n_before += __popc(bal);
            }
            if (lane == 0) a.qnbits[row] = n_before;
            if (alt == 0)
                for (int j = n_before + lane; j < kSlotBits; j += 32) s_bits[j] = 0;
        }
        if (lane == 0) {
            s_union[0] = u0;
            s_union[1] = u1;
        }
    }
    if (a.qscale != nullptr && threadIdx.x >= 32 && threadIdx.x < 64) {
        // bound of the query's scores, for the score bins of the scans and
        // the final top-k: |<q, x>| <= S = 128 * sum_j |q_j| for any int8 row x
        const int lane = threadIdx.x - 32;
        const int8_t* qv = a.queries + int64_t(b) * a.d;
        int32_t sum = 0;
        for (int j = lane; j < a.d; j += 32) sum += abs(int32_t(qv[j]));
        sum = __reduce_add_sync(0xffffffffu, sum);
        if (lane == 0) {
            const int32_t S = 128 * sum;
            int sh = 0;
            while (((int64_t(2) * S) >> sh) >= kTcBins) ++sh;
            a.qscale[b] = make_int2(-S, sh);
        }
    }
    __syncthreads();  // s_bits holds the query's first mask bits, s_union its masks' union
    const uint4 sb0 = reinterpret_cast<const uint4*>(s_bits)[0], sb1 = reinterpret_cast<const uint4*>(s_bits)[1];
    for (int p = threadIdx.x; p < P; p += BLOCK) {
        const int L = int(key_id(sorted[p]));
        a.probe[int64_t(b) * P + p] = L;
        if (L >= 0 && L < a.nlist) {
            const int r = atomicAdd(&a.list_cnt[L], 1);
            const int64_t slot = int64_t(L) * a.B + r;
            a.qlist[slot] = b;
            // the union of the query's masks: the planes its units need
            reinterpret_cast<ulonglong2*>(a.qmask_slot)[slot] = make_ulonglong2(s_union[0], s_union[1]);
            uint4* sbits = reinterpret_cast<uint4*>(a.slot_bits + slot * kSlotBits);
            sbits[0] = sb0;
            sbits[1] = sb1;
        }
    }
}

// Select query b's P best of the n keys (radix threshold), sort them, and
// write its probe result (file_query).
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
    file_query<BLOCK, kFile>(a, b, sortbuf);
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

// ----------------------------------------------------------------------------
// Search probe: tile scoring + per-query histogram-guided selection
// ----------------------------------------------------------------------------
constexpr int kTileC = 64;   // centroids per scoring CTA (one per thread of a query group)
constexpr int kTileQ = 64;   // queries per scoring CTA
constexpr int kQPer = 16;    // queries per thread
constexpr int kScoreBlock = kTileC * (kTileQ / kQPer);

__global__ void __launch_bounds__(kScoreBlock)
probe_score_kernel(SearchArgs a)
{
    // the selection kernel may start its query-only prologue meanwhile
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    extern __shared__ __align__(16) unsigned char smem_raw[];
    int4* sq = reinterpret_cast<int4*>(smem_raw);  // [kTileQ][np]
    const int d = a.d, np = d >> 4, nlist = a.nlist;
    const int c0 = blockIdx.x * kTileC, q0 = blockIdx.y * kTileQ;
    const int nq = a.B - q0 < kTileQ ? a.B - q0 : kTileQ;
    const int4* qsrc = reinterpret_cast<const int4*>(a.queries + int64_t(q0) * d);
    for (int i = threadIdx.x; i < nq * np; i += kScoreBlock) sq[i] = qsrc[i];
    __syncthreads();
    const int c = c0 + (threadIdx.x % kTileC);
    const int g = threadIdx.x / kTileC;  // this thread's queries: g*kQPer ..
    if (c >= nlist || g * kQPer >= nq) return;
    const int4* crow = reinterpret_cast<const int4*>(a.centroids + int64_t(c) * d);
    const int4* qg = sq + g * kQPer * np;
    int32_t acc[kQPer];
#pragma unroll
    for (int j = 0; j < kQPer; ++j) acc[j] = 0;
    for (int p = 0; p < np; ++p) {
        const int4 cv = __ldg(crow + p);
#pragma unroll
        for (int j = 0; j < kQPer; ++j) acc[j] = dot16(cv, qg[j * np + p], acc[j]);  // (rows past nq unused)
    }
    const int64_t ld = probe_keys_ld(nlist);
    uint64_t* out = a.probe_keys + int64_t(q0 + g * kQPer) * ld + c;
#pragma unroll
    for (int j = 0; j < kQPer; ++j)
        if (g * kQPer + j < nq) out[int64_t(j) * ld] = pack_key(acc[j], uint32_t(c));
}

// One cluster of CS CTAs per query: the nprobe best keys of the query's row
// of centroid keys (cluster_topk.cuh), then its probe result and filing.
constexpr int kProbeCBlock = 512;
constexpr int kProbeTieCap = 1024;

template <int CS>
__global__ void __launch_bounds__(kProbeCBlock)
probe_select_cluster_kernel(SearchArgs a)
{
    cooperative_groups::cluster_group cluster = cooperative_groups::this_cluster();
    const int b = int(blockIdx.x) / CS;
    const int P = a.P;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ SelectSmem ss;
    __shared__ ClusterCut cc;
    // shared layout: [tmp: P keys, rounded up to even][tie: kProbeTieCap keys][out: next_pow2(P) keys]
    uint64_t* tmp = reinterpret_cast<uint64_t*>(smem_raw);
    uint64_t* tie = tmp + ((P + 1) & ~1);
    uint64_t* out = tie + kProbeTieCap;
    const uint64_t* row = a.probe_keys + int64_t(b) * probe_keys_ld(a.nlist);
    // every centroid score lies in [-Sc, Sc], Sc = 128 sum_j |q_j| (int8
    // centroids), so the selection needs no pass over the keys for their range
    __shared__ int32_t s_sc;
    __shared__ uint32_t s_hits[4];
    // the query's expected selectivity (sample rows passing any of its masks),
    // counted by the leader CTA's warps 1 to 4 while warp 0 sums |q|
    const bool count_sel = a.qsel != nullptr && int(blockIdx.x) % CS == 0;
    static_assert(kSelSample % 128 == 0 && 32 + 128 <= kProbeCBlock, "four warps hold the sample");
    if (threadIdx.x < 32) {
        int32_t sum = 0;
        for (int j = threadIdx.x; j < a.d; j += 32) sum += abs(int32_t(a.queries[int64_t(b) * a.d + j]));
        sum = __reduce_add_sync(0xffffffffu, sum);
        if (threadIdx.x == 0) s_sc = 128 * sum;
    } else if (count_sel && threadIdx.x < 32 + 128) {
        constexpr int kRows = kSelSample / 128;  // sample rows per thread
        const int t = threadIdx.x - 32, W = a.W;
        uint64_t s0[kRows], s1[kRows];
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            const int i = t + 128 * r;
            s0[r] = i < a.n_sample ? a.sig_sample[int64_t(i) * W] : 0ull;
            s1[r] = i < a.n_sample && W > 1 ? a.sig_sample[int64_t(i) * W + 1] : 0ull;
        }
        uint32_t pass = 0;  // bit r: row t + 128 r passes one of the masks
        for (int alt = 0; alt <= a.n_or; ++alt) {
            const uint64_t* mk = alt == 0 ? a.qmasks + int64_t(b) * W : a.or_masks + (int64_t(b) * a.n_or + alt - 1) * W;
            const uint64_t m0 = mk[0], m1 = W > 1 ? mk[1] : 0ull;
#pragma unroll
            for (int r = 0; r < kRows; ++r)
                if (t + 128 * r < a.n_sample && (s0[r] & m0) == m0 && (s1[r] & m1) == m1) pass |= 1u << r;
        }
        const uint32_t hits = __reduce_add_sync(0xffffffffu, uint32_t(__popc(pass)));
        if ((threadIdx.x & 31) == 0) s_hits[(threadIdx.x >> 5) - 1] = hits;
    }
    __syncthreads();
    if (count_sel && threadIdx.x == 0) {
        const uint32_t h = s_hits[0] + s_hits[1] + s_hits[2] + s_hits[3];
        a.qsel[b] = uint16_t(h);
        atomicMax(reinterpret_cast<unsigned int*>(&a.ctl->max_qsel), h);  // lets the plan skip hopeless lists
    }
    // everything above reads the query, its masks and the index only (and
    // writes scratch the search's memset cleared before the scoring kernel
    // started), so it ran while the scoring kernel was still working
    dep_enter();
    const int32_t sc = s_sc;
    auto none = [](uint64_t) { return true; };
    auto no_compact = []() { return 0; };
    const int m = cluster_topk<CS, kProbeCBlock>(cluster, row, a.nlist, P, true, -sc, sc, false, none, no_compact, tmp,
                                                 tie, kProbeTieCap, out, ss, cc, a.err);
    if (m < 0) return;  // not the leader
    if (threadIdx.x == 0 && m != P) set_error(a.err, kErrSelectCount);
    file_query<kProbeCBlock, true>(a, b, out);
}

static size_t probe_select_smem(int P)
{
    return (size_t((P + 1) & ~1) + kProbeTieCap + size_t(next_pow2(P))) * 8;
}

template <int CS>
static cudaError_t launch_probe_select(const SearchArgs& a, cudaStream_t s)
{
    const void* fn = reinterpret_cast<const void*>(probe_select_cluster_kernel<CS>);
    cudaError_t e = ensure_smem_attr(fn, int(probe_select_smem(ST_MAX_NPROBE)));
    if (e != cudaSuccess) return e;
    return launch_dep_cluster(probe_select_cluster_kernel<CS>, dim3(unsigned(a.B) * CS), dim3(kProbeCBlock),
                              probe_select_smem(a.P), CS, s, a);
}

cudaError_t launch_probe_search(const SearchArgs& a, int num_sms, cudaStream_t s)
{
    const dim3 grid((a.nlist + kTileC - 1) / kTileC, (a.B + kTileQ - 1) / kTileQ);
    const size_t qbytes = size_t(kTileQ) * a.d;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(probe_score_kernel), int(kTileQ * ST_MAX_D));
    if (e != cudaSuccess) return e;
    probe_score_kernel<<<grid, kScoreBlock, qbytes, s>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    switch (cluster_size_for(a.B, num_sms)) {
    case 8: return launch_probe_select<8>(a, s);
    case 4: return launch_probe_select<4>(a, s);
    case 2: return launch_probe_select<2>(a, s);
    default: return launch_probe_select<1>(a, s);
    }
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
    e = ensure_smem_attr(reinterpret_cast<const void*>(probe_kernel<kProbeBlock, false>), 200 * 1024);
    if (e != cudaSuccess) return e;
    probe_kernel<kProbeBlock, false><<<a.B * S, kProbeBlock, smem, s>>>(a, S);
    return cudaGetLastError();
}

}  // namespace st
