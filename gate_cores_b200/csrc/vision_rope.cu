// Vision 2-D RoPE of the NaViT tower (page "...muse_spark.vision":
// _apply_vision_rope, _rope_frequencies).
//
// Rotation: one warp per token walks the token's Q then K vectors (16 bytes
// each, heads contiguous within a token) with a lane stride that is a
// multiple of the vectors per head (nvh): lane L only ever meets position
// L mod nvh of a head, so the (cos, sin) pairs of that position - the same
// for every head of the token - are loaded once into registers (lanes
// stride..31 idle; 30 of 32 lanes for heads of 80 bf16).  Each lane issues
// the loads of B vectors before rotating adjacent pairs in FP32
//   y[2i] = a c - b s,   y[2i+1] = a s + b c,
// and writes the results cast to the Q/K dtype.  Exact in-place (q_out == q)
// is safe: a lane writes only the vectors it has read.  Heads of at most 32
// vectors (512 bytes).
//
// Table: one thread per (patch, pair) of a row-major grid; the first
// head_dim/4 pairs take the patch row, the others the column, angle =
// f32(coord) * inv_freq[j] (one FP32 rounding), sincosf of it.
#include "common.cuh"
#include "kernels.h"

namespace muse {
namespace {

constexpr int kVisionThreads = 256;
constexpr int kVisionBatch = 6;  // measured: 8 and 4 slower (register pressure / too few loads in flight)

template <typename T>
__global__ void __launch_bounds__(kVisionThreads, 4) vision_rope_kernel(const __grid_constant__ VisionRopeArgs a) {
    pdl_begin();
    constexpr int V = Vec<T>::N;
    constexpr int B = kVisionBatch;
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * (kVisionThreads / 32) + (threadIdx.x >> 5);
    const int nvh = a.head_dim / V;           // 16-byte vectors per head, 1 .. 32
    const int stride = (32 / nvh) * nvh;      // lanes in use
    if (t >= a.tokens || lane >= stride) return;
    const int nq = a.hq * nvh;
    const int nv = nq + a.hk * nvh;
    const char* q = static_cast<const char*>(a.q) + t * a.q_stride * (int64_t)sizeof(T);
    const char* k = static_cast<const char*>(a.k) + t * a.k_stride * (int64_t)sizeof(T);
    char* qo = static_cast<char*>(a.q_out) + t * a.q_out_stride * (int64_t)sizeof(T);
    char* ko = static_cast<char*>(a.k_out) + t * a.k_out_stride * (int64_t)sizeof(T);
    // (cos, sin) of the V/2 pairs at this lane's position within a head
    float4 cs[V / 4];
    {
        const float4* f4 = reinterpret_cast<const float4*>(a.freqs + t * (int64_t)a.head_dim + (lane % nvh) * V);
#pragma unroll
        for (int p = 0; p < V / 4; ++p) cs[p] = __ldg(f4 + p);
    }
#pragma unroll 1
    for (int v0 = lane; v0 < nv; v0 += stride * B) {
        uint4 xv[B];
#pragma unroll
        for (int u = 0; u < B; ++u) {
            const int v = v0 + stride * u;
            if (v < nv) xv[u] = ld_stream(v < nq ? q + (size_t)v * 16u : k + (size_t)(v - nq) * 16u);
        }
#pragma unroll
        for (int u = 0; u < B; ++u) {
            const int v = v0 + stride * u;
            if (v >= nv) break;
            float x[V], y[V];
            unpack<T>(xv[u], x);
#pragma unroll
            for (int p = 0; p < V / 4; ++p) {  // float4 p holds the (c, s) of pairs 2p, 2p + 1
                const float4 c4 = cs[p];
                const float a0 = x[4 * p], b0 = x[4 * p + 1], a1 = x[4 * p + 2], b1 = x[4 * p + 3];
                y[4 * p] = fmaf(-b0, c4.y, a0 * c4.x);
                y[4 * p + 1] = fmaf(a0, c4.y, b0 * c4.x);
                y[4 * p + 2] = fmaf(-b1, c4.w, a1 * c4.z);
                y[4 * p + 3] = fmaf(a1, c4.w, b1 * c4.z);
            }
            st_vec(v < nq ? qo + (size_t)v * 16u : ko + (size_t)(v - nq) * 16u, pack<T>(y));
        }
    }
}

__global__ void __launch_bounds__(kVisionThreads) vision_rope_frequencies_kernel(const __grid_constant__ VisionFreqArgs a) {
    pdl_begin();
    const int half = a.head_dim / 2, quarter = a.head_dim / 4;
    const int64_t n = (int64_t)a.grid_h * a.grid_w * half;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n; idx += (int64_t)gridDim.x * blockDim.x) {
        const int i = (int)(idx % half);
        const int64_t p = idx / half;
        const int h = (int)(p / a.grid_w), w = (int)(p % a.grid_w);
        const float coord = (float)(i < quarter ? h : w);
        const float phi = coord * a.inv_freq[i < quarter ? i : i - quarter];  // one FP32 rounding
        float s, c;
        sincosf(phi, &s, &c);
        reinterpret_cast<float2*>(a.out)[idx] = make_float2(c, s);
    }
}

}  // namespace

cudaError_t launch_vision_rope(int dtype, const VisionRopeArgs& a, cudaStream_t s) {
    const int64_t per_cta = kVisionThreads / 32;
    const unsigned grid = (unsigned)((a.tokens + per_cta - 1) / per_cta);
    return dtype == 0 ? launch_pdl(vision_rope_kernel<__nv_bfloat16>, grid, kVisionThreads, 0, s, a)
                      : launch_pdl(vision_rope_kernel<float>, grid, kVisionThreads, 0, s, a);
}

cudaError_t launch_vision_rope_frequencies(const VisionFreqArgs& a, cudaStream_t s) {
    const int64_t n = (int64_t)a.grid_h * a.grid_w * (a.head_dim / 2);
    int64_t grid = (n + kVisionThreads - 1) / kVisionThreads;
    if (grid > 65535) grid = 65535;
    return launch_pdl(vision_rope_frequencies_kernel, (unsigned)grid, kVisionThreads, 0, s, a);
}

}  // namespace muse
