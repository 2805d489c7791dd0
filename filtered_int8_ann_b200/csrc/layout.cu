// Index layout: Bloom signatures as bit-planes per list chunk.
//
// The Bloom test of the method -- every bit of the request mask present in the
// item's signature (SilverTorch: Index as Model, section on redesigning each
// stage as a pure PyTorch module, Bloom index filter paragraph) -- only ever
// looks at the signature bits the mask sets, and a request mask sets few of
// them (about 18 of 128 for a language, a country and four flags at three bits
// each). Row-major signatures make the scan read all 128 bits of every item.
//
// Here each list chunk (kWarpItems consecutive rows of one list, the scan's
// unit of work) stores its signatures transposed: plane b of chunk t is
// kWarpItems bits = 16 words, bit i of word w being bit b of row 32w + i of the
// chunk (rows past the end of the list are zero). A scan unit then fetches only
// the planes of the bits its queries' masks use, and tests 32 items with one
// 32-bit AND per mask bit.
//
// Inserted items go to append chunks: blocks of kWarpItems rows after all the
// creation rows, each owned by one list and filled in order; their planes
// follow the creation chunks' planes. The search walks a list chunk by chunk
// through a descriptor table, so a list's creation rows and append chunks need
// not be adjacent.
#include "st_internal.cuh"

namespace st {

// One warp per (chunk, 32-row block): each lane holds one row's signature and
// every plane word comes out of one warp ballot.
template <int W>
__global__ void __launch_bounds__(256)
build_planes_kernel(const uint64_t* __restrict__ sigs, const int64_t* __restrict__ offsets,
                    const int32_t* __restrict__ chunk_start, const int32_t* __restrict__ chunk_list,
                    int32_t n_chunks, uint32_t* __restrict__ planes)
{
    constexpr int NPL = 64 * W;
    const int lane = threadIdx.x & 31;
    const int64_t g = (int64_t(blockIdx.x) * 256 + threadIdx.x) >> 5;  // warp id
    if (g >= int64_t(n_chunks) * 16) return;
    const int t = int(g >> 4), w = int(g & 15);
    const int L = chunk_list[t];
    const int c = t - chunk_start[L];
    const int64_t first = offsets[L] + int64_t(c) * kWarpItems;
    const int64_t end = min(offsets[L + 1], first + kWarpItems);
    const int64_t row = first + 32 * w + lane;
    uint64_t s0 = 0, s1 = 0;
    if (row < end) {
        s0 = sigs[row * W];
        if (W > 1) s1 = sigs[row * W + 1];
    }
    uint32_t* dst = planes + int64_t(t) * NPL * 16 + w;
#pragma unroll 8
    for (int b = 0; b < NPL; ++b) {
        const uint64_t word = b < 64 ? s0 : s1;
        const unsigned bal = __ballot_sync(0xffffffffu, (word >> (b & 63)) & 1ull);
        if (lane == (b & 31)) dst[b * 16] = bal;
    }
}

// The plane block of item `id` and its row within the block; false for an id
// the index never handed out.
__device__ __forceinline__ bool locate_row(const RowMap& map, int64_t id, int64_t& block, int& r)
{
    if (id < 0) return false;
    if (id < map.n) {
        // the row's list: the last c with offsets[c] <= id (empty lists share offsets)
        int lo = 0, hi = map.nlist - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (map.offsets[mid] <= id) lo = mid;
            else hi = mid - 1;
        }
        const int64_t rr = id - map.offsets[lo];
        block = map.base_chunk_start[lo] + rr / kWarpItems;
        r = int(rr % kWarpItems);
        return true;
    }
    const int64_t a = (id - map.n) / kWarpItems;
    if (a >= map.n_app) return false;
    r = int((id - map.n) % kWarpItems);
    if (r >= map.app_len[a]) return false;
    block = map.n_base_chunks + a;
    return true;
}

// In-place update (and insertion) of m rows: one warp per row copies the new
// row and signature and rewrites the row's bit in each of its chunk's planes
// (atomically: other rows of the same plane words may change at the same time).
template <int W>
__global__ void __launch_bounds__(256)
update_kernel(int8_t* items, uint64_t* sigs, uint32_t* planes, RowMap map, int d, const int64_t* ids,
              const int8_t* new_items, const uint64_t* new_sigs, int64_t m, uint32_t* err)
{
    constexpr int NPL = 64 * W;
    const int lane = threadIdx.x & 31;
    const int64_t j = (int64_t(blockIdx.x) * 256 + threadIdx.x) >> 5;
    if (j >= m) return;
    const int64_t id = ids[j];
    int64_t t = 0;
    int r = 0;
    if (!locate_row(map, id, t, r)) {
        if (lane == 0) atomicOr(err, kErrUpdateId);
        return;
    }
    if (new_items)
        for (int p = lane; p < d / 16; p += 32)
            reinterpret_cast<int4*>(items + id * d)[p] = reinterpret_cast<const int4*>(new_items + j * d)[p];
    if (!new_sigs) return;
    const int w = r >> 5;
    const uint32_t bit = 1u << (r & 31);
    uint64_t s0 = new_sigs[j * W], s1 = W > 1 ? new_sigs[j * W + 1] : 0ull;
    if (lane == 0) {
        sigs[id * W] = s0;
        if (W > 1) sigs[id * W + 1] = s1;
    }
    uint32_t* pl = planes + t * NPL * 16 + w;
    for (int b = lane; b < NPL; b += 32) {
        const bool on = ((b < 64 ? s0 : s1) >> (b & 63)) & 1ull;
        if (on) atomicOr(pl + b * 16, bit);
        else atomicAnd(pl + b * 16, ~bit);
    }
}

// Deletion: one thread per id sets the item's bit in the deletion bitmap.
__global__ void __launch_bounds__(256)
delete_kernel(uint32_t* dead, RowMap map, const int64_t* ids, int64_t m, uint32_t* err)
{
    const int64_t j = int64_t(blockIdx.x) * 256 + threadIdx.x;
    if (j >= m) return;
    const int64_t id = ids[j];
    int64_t t = 0;
    int r = 0;
    if (!locate_row(map, id, t, r)) {
        atomicOr(err, kErrUpdateId);
        return;
    }
    atomicOr(dead + (id >> 5), 1u << (id & 31));
}

cudaError_t launch_delete(uint32_t* dead, const RowMap& map, const int64_t* ids, int64_t m, uint32_t* err,
                          cudaStream_t s)
{
    if (m <= 0) return cudaSuccess;
    delete_kernel<<<unsigned((m + 255) / 256), 256, 0, s>>>(dead, map, ids, m, err);
    return cudaGetLastError();
}

cudaError_t launch_update(int8_t* items, uint64_t* sigs, uint32_t* planes, const RowMap& map, int d, int W,
                          const int64_t* ids, const int8_t* new_items, const uint64_t* new_sigs, int64_t m,
                          uint32_t* err, cudaStream_t s)
{
    if (m <= 0) return cudaSuccess;
    const int64_t blocks = (m * 32 + 255) / 256;
    if (W == 2)
        update_kernel<2><<<unsigned(blocks), 256, 0, s>>>(items, sigs, planes, map, d, ids, new_items, new_sigs, m,
                                                          err);
    else
        update_kernel<1><<<unsigned(blocks), 256, 0, s>>>(items, sigs, planes, map, d, ids, new_items, new_sigs, m,
                                                          err);
    return cudaGetLastError();
}

cudaError_t launch_build_planes(const uint64_t* sigs, const int64_t* offsets, const int32_t* chunk_start,
                                const int32_t* chunk_list, int32_t n_chunks, int W, uint32_t* planes,
                                cudaStream_t s)
{
    const int64_t warps = int64_t(n_chunks) * 16;
    const int64_t blocks = (warps * 32 + 255) / 256;
    if (blocks <= 0) return cudaSuccess;
    if (W == 2)
        build_planes_kernel<2><<<unsigned(blocks), 256, 0, s>>>(sigs, offsets, chunk_start, chunk_list, n_chunks, planes);
    else
        build_planes_kernel<1><<<unsigned(blocks), 256, 0, s>>>(sigs, offsets, chunk_start, chunk_list, n_chunks, planes);
    return cudaGetLastError();
}

}  // namespace st
