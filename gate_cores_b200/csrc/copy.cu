// 16-byte vector copy over a persistent grid: the HBM bandwidth reference the
// cores are measured against (read + write bytes / time).
#include "common.cuh"
#include "kernels.h"

namespace muse {
namespace {

constexpr int kUnroll = 4;

__global__ void __launch_bounds__(512) copy_kernel(const uint4* __restrict__ src,
                                                   uint4* __restrict__ dst, int64_t n) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    // kUnroll independent loads in flight per thread, then their stores.
    for (; i + (kUnroll - 1) * stride < n; i += kUnroll * stride) {
        uint4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) v[u] = ld_stream(src + i + u * stride);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) st_vec(dst + i + u * stride, v[u]);
    }
    for (; i < n; i += stride) st_vec(dst + i, ld_stream(src + i));
}

}  // namespace

cudaError_t launch_copy(const void* src, void* dst, int64_t bytes, cudaStream_t s) {
    const int64_t n = bytes / 16;
    const int threads = 512;
    int64_t grid = (int64_t)blocks_per_sm((const void*)copy_kernel, threads) * sm_count();
    const int64_t need = (n + threads - 1) / threads;
    if (grid > need) grid = need;
    if (grid < 1) grid = 1;
    copy_kernel<<<(unsigned)grid, threads, 0, s>>>(static_cast<const uint4*>(src),
                                                   static_cast<uint4*>(dst), n);
    return cudaGetLastError();
}

}  // namespace muse
