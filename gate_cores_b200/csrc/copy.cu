// 16-byte vector copy: the HBM bandwidth reference the cores are measured
// against (read + write bytes / time).  One-shot grid: each CTA copies one
// contiguous tile of kThreads x kUnroll vectors (all loads first, then the
// stores) and exits, so at any time the resident CTAs stream one compact
// window of memory.  Measured on B200 (1 GiB): about 6.8 TB/s, against 5.8
// TB/s for a persistent grid-stride loop whose loads in flight lie a whole
// grid apart.
#include "common.cuh"
#include "kernels.h"

namespace muse {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

__global__ void __launch_bounds__(kThreads) copy_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                        int64_t n) {
    pdl_begin();
    const int64_t base = (int64_t)blockIdx.x * (kThreads * kUnroll) + threadIdx.x;
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + (int64_t)u * kThreads;
        if (i < n) v[u] = ld_stream(src + i);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + (int64_t)u * kThreads;
        if (i < n) st_vec(dst + i, v[u]);
    }
}

}  // namespace

cudaError_t launch_copy(const void* src, void* dst, int64_t bytes, cudaStream_t s) {
    const int64_t n = bytes / 16;
    const int64_t grid = (n + kThreads * kUnroll - 1) / (kThreads * kUnroll);
    if (grid > 0x7fffffff) return cudaErrorInvalidValue;
    return launch_pdl(copy_kernel, (unsigned)(grid < 1 ? 1 : grid), (unsigned)kThreads, 0, s,
                      static_cast<const uint4*>(src), static_cast<uint4*>(dst), n);
}

}  // namespace muse
