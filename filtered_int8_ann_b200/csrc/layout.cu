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
