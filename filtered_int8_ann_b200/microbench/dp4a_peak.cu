// Microbenchmark of the dp4a issue rate: the ALU ceiling of the scan's int8
// inner products when they are not on the tensor cores. It only launches a
// kernel and times it with CUDA events; it reads and changes no GPU setting.
//
// Every thread runs kChains independent dp4a accumulation chains for `iters`
// steps; operands change every step so nothing can be folded, and the sums
// are stored so nothing is dead. One dp4a = 4 multiplies + 4 adds = 8 int8
// operations, the same count as 2 * d operations per d-dimensional score.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

constexpr int kChains = 8;
constexpr int kBlock = 256;

__global__ void __launch_bounds__(kBlock) dp4a_loop(int iters, int seed, int32_t* out)
{
    int32_t acc[kChains];
    int a[kChains], b[kChains];
#pragma unroll
    for (int c = 0; c < kChains; ++c) {
        acc[c] = c;
        a[c] = seed * (c + 1) + int(threadIdx.x);
        b[c] = seed ^ (0x01010101 * (c + 3)) ^ int(blockIdx.x);
    }
    for (int i = 0; i < iters; ++i) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
#pragma unroll
            for (int c = 0; c < kChains; ++c) acc[c] = __dp4a(a[c], b[c], acc[c]);
        }
#pragma unroll
        for (int c = 0; c < kChains; ++c) a[c] += 0x01020304;
    }
    int32_t s = 0;
#pragma unroll
    for (int c = 0; c < kChains; ++c) s ^= acc[c];
    out[blockIdx.x * kBlock + threadIdx.x] = s;
}

}  // namespace

extern "C" {

// Measured dp4a throughput of the current device, in int8 TOPS (10^12 int8
// operations per second), the best of `reps` timed launches after two
// warm-ups. Grid: 8 blocks of 256 threads per SM. Returns 0 on success, else
// the CUDA error code.
int st_peak_dp4a_tops(int reps, double* tops)
{
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return int(e);
    const int grid = sms * 8;
    const int iters = 4096;
    int32_t* out = nullptr;
    cudaEvent_t t0 = nullptr, t1 = nullptr;
    e = cudaMalloc(&out, size_t(grid) * kBlock * sizeof(int32_t));
    if (e == cudaSuccess) e = cudaEventCreate(&t0);
    if (e == cudaSuccess) e = cudaEventCreate(&t1);
    float best = 0.f;
    for (int r = 0; e == cudaSuccess && r < reps + 2; ++r) {
        cudaEventRecord(t0);
        dp4a_loop<<<grid, kBlock>>>(iters, r + 1, out);
        cudaEventRecord(t1);
        e = cudaEventSynchronize(t1);
        float ms = 0.f;
        if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, t0, t1);
        if (e == cudaSuccess && r >= 2 && (best == 0.f || ms < best)) best = ms;
    }
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e == cudaSuccess && best > 0.f) {
        const double ops = double(grid) * kBlock * iters * 4.0 * kChains * 8.0;
        *tops = ops / (double(best) * 1e-3) / 1e12;
    }
    if (t0) cudaEventDestroy(t0);
    if (t1) cudaEventDestroy(t1);
    cudaFree(out);
    return int(e);
}

}  // extern "C"
