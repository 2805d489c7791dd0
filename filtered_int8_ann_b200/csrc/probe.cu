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
// One CTA per query. The query's int8 words sit in shared memory (every thread
// reads the same word: a broadcast); each thread streams whole centroid rows
// with 16-byte read-only loads and accumulates with dp4a. The centroid table
// (nlist * d bytes, 1 MiB for 16384 x 64) stays L2-resident across CTAs. Keys
// stay in shared memory up to 16384 lists and spill to a global scratch row
// beyond, then an in-CTA radix select picks the nprobe best keys. Each chosen
// list bumps its query count, which the plan kernel consumes.
#include "st_internal.cuh"

namespace st {

template <int BLOCK>
__global__ void __launch_bounds__(BLOCK)
probe_kernel(SearchArgs a)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ SelectSmem ss;
    const int b = blockIdx.x;
    const int d = a.d;
    const int nlist = a.nlist;
    const int P = a.P;
    const int pw = next_pow2(P);
    const int pws = pw < 2 ? 2 : pw;

    // shared layout: [sort buffer pws keys][query d bytes][keys nlist (if local)]
    uint64_t* sortbuf = reinterpret_cast<uint64_t*>(smem_raw);
    int4* qv = reinterpret_cast<int4*>(sortbuf + pws);
    const bool local_keys = (a.probe_keys == nullptr);
    uint64_t* keys = local_keys ? reinterpret_cast<uint64_t*>(qv + d / 16)
                                : a.probe_keys + int64_t(b) * nlist;

    const int4* q4 = reinterpret_cast<const int4*>(a.queries + int64_t(b) * d);
    for (int j = threadIdx.x; j < d / 16; j += BLOCK) qv[j] = q4[j];
    __syncthreads();

    const int np = d / 16;
    for (int c = threadIdx.x; c < nlist; c += BLOCK) {
        const int4* row = reinterpret_cast<const int4*>(a.centroids + int64_t(c) * d);
        int32_t acc = 0;
        for (int p = 0; p < np; ++p) acc = dot16(__ldg(row + p), qv[p], acc);
        keys[c] = pack_key(acc, uint32_t(c));
    }
    __syncthreads();

    uint64_t thr = 0;
    if (P < nlist) thr = block_select_threshold<BLOCK>(keys, nlist, P, ss, a.err);
    const int got = block_collect_ge<BLOCK>(keys, nlist, thr, sortbuf, pw, ss);
    if (threadIdx.x == 0 && got != P) set_error(a.err, kErrSelectCount);
    for (int i = (got < pw ? got : pw) + threadIdx.x; i < pw; i += BLOCK) sortbuf[i] = 0;
    __syncthreads();
    block_bitonic_desc<BLOCK>(sortbuf, pw);
    for (int p = threadIdx.x; p < P; p += BLOCK) {
        const int L = int(key_id(sortbuf[p]));
        a.probe[int64_t(b) * P + p] = L;
        if (L >= 0 && L < nlist) atomicAdd(&a.list_cnt[L], 1);
    }
}

static size_t probe_smem_bytes(const SearchArgs& a)
{
    const int pw = next_pow2(a.P);
    size_t bytes = size_t(pw < 2 ? 2 : pw) * 8 + size_t(a.d);
    if (a.probe_keys == nullptr) bytes += size_t(a.nlist) * 8;
    return bytes;
}

cudaError_t launch_probe(const SearchArgs& a, cudaStream_t s)
{
    const size_t smem = probe_smem_bytes(a);
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(probe_kernel<kProbeBlock>), 0, 200 * 1024);
    if (e != cudaSuccess) return e;
    probe_kernel<kProbeBlock><<<a.B, kProbeBlock, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace st
