// Device helpers shared by the normalisation kernels: 16-byte vector memory
// access, bf16 <-> FP32 conversion and warp / CTA reductions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace muse {

// Elements of T in one 16-byte vector.
template <typename T> struct Vec;
template <> struct Vec<__nv_bfloat16> { static constexpr int N = 8; };
template <> struct Vec<float> { static constexpr int N = 4; };

// Programmatic dependent launch.  Every kernel of the library starts with
// pdl_begin(): it lets the next kernel of the stream begin launching (its CTAs
// take SM slots as this grid's CTAs retire), then waits until the previous
// kernel of the stream has completed and its writes are visible.  Nothing is
// read or written before the wait.  Both instructions are no-ops in a launch
// without the programmatic-serialization attribute.
__device__ __forceinline__ void pdl_begin() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Launch with programmatic stream serialization allowed (the kernel must
// begin with pdl_begin()).  Returns the launch error.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Streaming 16-byte load: cached in L2 only (every input byte is read once).
__device__ __forceinline__ uint4 ld_stream(const void* p) {
    return __ldcg(reinterpret_cast<const uint4*>(p));
}

// 16-byte store.
__device__ __forceinline__ void st_vec(void* p, const uint4& v) {
    *reinterpret_cast<uint4*>(p) = v;
}

// bf16 pair held in one 32-bit word -> two floats (exact).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Two floats -> bf16 pair, round to nearest even (cvt.rn.bf16x2.f32).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Round a float to the nearest bf16 value and return it as a float.
__device__ __forceinline__ float round_bf16(float v) {
    return __bfloat162float(__float2bfloat16_rn(v));
}

// Round to the activation dtype (identity for FP32).
template <typename T> __device__ __forceinline__ float round_to(float v);
template <> __device__ __forceinline__ float round_to<__nv_bfloat16>(float v) { return round_bf16(v); }
template <> __device__ __forceinline__ float round_to<float>(float v) { return v; }

// 16-byte vector <-> Vec<T>::N floats.
template <typename T> __device__ __forceinline__ void unpack(const uint4& v, float* f);
template <> __device__ __forceinline__ void unpack<__nv_bfloat16>(const uint4& v, float* f) {
    f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
    f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
    f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
    f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}
template <> __device__ __forceinline__ void unpack<float>(const uint4& v, float* f) {
    f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
}

template <typename T> __device__ __forceinline__ uint4 pack(const float* f);
template <> __device__ __forceinline__ uint4 pack<__nv_bfloat16>(const float* f) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                      pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
}
template <> __device__ __forceinline__ uint4 pack<float>(const float* f) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]),
                      __float_as_uint(f[2]), __float_as_uint(f[3]));
}

// ---- Packed FP32 pairs (Blackwell f32x2 instructions: one issue slot, two
// IEEE round-to-nearest FP32 operations, bit-identical to two scalar ones).
typedef unsigned long long f32x2;

__device__ __forceinline__ f32x2 f2_make(float lo, float hi) {
    f32x2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_split(f32x2 p, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(p));
}
__device__ __forceinline__ f32x2 f2_mul(f32x2 a, f32x2 b) {
    f32x2 r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ f32x2 f2_add(f32x2 a, f32x2 b) {
    f32x2 r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ f32x2 f2_fma(f32x2 a, f32x2 b, f32x2 c) {
    f32x2 r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

// A 16-byte vector of T as Vec<T>::N / 2 packed pairs (element order kept).
template <typename T> __device__ __forceinline__ void to_pairs(const uint4& v, f32x2* p);
template <> __device__ __forceinline__ void to_pairs<__nv_bfloat16>(const uint4& v, f32x2* p) {
    p[0] = f2_make(bf16_lo(v.x), bf16_hi(v.x));
    p[1] = f2_make(bf16_lo(v.y), bf16_hi(v.y));
    p[2] = f2_make(bf16_lo(v.z), bf16_hi(v.z));
    p[3] = f2_make(bf16_lo(v.w), bf16_hi(v.w));
}
template <> __device__ __forceinline__ void to_pairs<float>(const uint4& v, f32x2* p) {
    p[0] = f2_make(__uint_as_float(v.x), __uint_as_float(v.y));
    p[1] = f2_make(__uint_as_float(v.z), __uint_as_float(v.w));
}

// Pairs -> 16-byte vector of T (bf16: round to nearest even).
template <typename T> __device__ __forceinline__ uint4 from_pairs(const f32x2* p);
template <> __device__ __forceinline__ uint4 from_pairs<__nv_bfloat16>(const f32x2* p) {
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        float lo, hi;
        f2_split(p[k], lo, hi);
        w[k] = pack_bf16x2(lo, hi);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}
template <> __device__ __forceinline__ uint4 from_pairs<float>(const f32x2* p) {
    float a, b, c, d;
    f2_split(p[0], a, b);
    f2_split(p[1], c, d);
    return make_uint4(__float_as_uint(a), __float_as_uint(b), __float_as_uint(c), __float_as_uint(d));
}

// Round a pair to T and back (the cast at a dtype boundary; exact for FP32).
template <typename T> __device__ __forceinline__ f32x2 round_pair(f32x2 p);
template <> __device__ __forceinline__ f32x2 round_pair<__nv_bfloat16>(f32x2 p) {
    float lo, hi;
    f2_split(p, lo, hi);
    const uint32_t w = pack_bf16x2(lo, hi);
    return f2_make(bf16_lo(w), bf16_hi(w));
}
template <> __device__ __forceinline__ f32x2 round_pair<float>(f32x2 p) { return p; }

__device__ __forceinline__ float f2_sum(f32x2 p) {
    float lo, hi;
    f2_split(p, lo, hi);
    return lo + hi;
}

// Sum of squares of N floats as a balanced tree (short rounding chains).
template <int N> __device__ __forceinline__ float sum_sq(const float* f) {
    if constexpr (N == 1) {
        return f[0] * f[0];
    } else {
        return sum_sq<N / 2>(f) + sum_sq<N - N / 2>(f + N / 2);
    }
}

// Butterfly sum over groups of G consecutive lanes (G a power of two <= 32).
// Every lane of a group ends with the same bits: IEEE addition is commutative,
// so both partners of each exchange compute the same rounded sum.
template <int G> __device__ __forceinline__ float group_sum(float v) {
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Sum over the whole CTA (blockDim.x a multiple of 32).  `red` holds two
// banks of 32 partials used alternately, so consecutive calls need only one
// __syncthreads each.  Every thread returns the same bits.
__device__ __forceinline__ float block_sum(float v, float (*red)[32], int& bank) {
    v = group_sum<32>(v);
    const int nw = blockDim.x >> 5;
    if (nw == 1) return v;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[bank][warp] = v;
    __syncthreads();
    float t = lane < nw ? red[bank][lane] : 0.0f;
    bank ^= 1;
    return group_sum<32>(t);
}

// 1 / sqrt(mean + eps) with IEEE-rounded division and square root (row
// kernels: once per row per thread, so the cost is spread over the row).
__device__ __forceinline__ float inv_rms(float sum_sq_total, float width, float eps) {
    return 1.0f / sqrtf(sum_sq_total / width + eps);
}

// Per-head variant: rsqrtf (at most 2 ulp) on mean * (1/width) + eps.  Its
// error stays far below the 2^-20 margin the bf16 casts are checked with.
__device__ __forceinline__ float inv_rms_fast(float sum_sq_total, float inv_width, float eps) {
    return rsqrtf(sum_sq_total * inv_width + eps);
}

// Reciprocal of a normal number (rcp.approx.ftz.f32, at most 1 ulp).
__device__ __forceinline__ float rcp_approx_ftz(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// 2^x (ex2.approx.ftz.f32).
__device__ __forceinline__ float exp2_approx(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// v * sigmoid(g), sigmoid(g) = 1 / (1 + exp(-g)), in FP32 without losing
// results that fall below the FP32 normal range.  With a = |g| and
// t = 2^64 exp(-a) (normal for a < 132, using exp(x) = 2^(x log2 e)):
//   g >= 0: sigmoid = 1 / (1 + t 2^-64);
//   g <  0: sigmoid = exp(g) / (1 + exp(g)) = t 2^-64 / (1 + t 2^-64),
// and the 2^-64 is applied last, so a subnormal product is rounded once.
// Relative error about 1e-5 for |g| ~ 100, far inside a bf16 output ulp.
template <typename T> __device__ __forceinline__ float times_sigmoid(float v, float g);
template <> __device__ __forceinline__ float times_sigmoid<__nv_bfloat16>(float v, float g) {
    const float a = fabsf(g);
    const float t = exp2_approx(fmaf(-a, 1.44269504088896341f, 64.0f));
    // 1 + t 2^-64 lies in [1, 2]: the flush-to-zero reciprocal is exact enough.
    const float d = rcp_approx_ftz(fmaf(t, 0x1p-64f, 1.0f));
    return g >= 0.0f ? v * d : ((v * t) * d) * 0x1p-64f;
}
// FP32 outputs need FP32 accuracy: expf (at most 2 ulp) and IEEE division;
// below exp(-80) the exponent is shifted by an exactly representable 64 and
// exp(-64) is applied last.
template <> __device__ __forceinline__ float times_sigmoid<float>(float v, float g) {
    const float a = fabsf(g);
    if (a <= 80.0f) {
        const float t = expf(-a);
        const float d = 1.0f / (1.0f + t);
        return g >= 0.0f ? v * d : (v * t) * d;
    }
    if (g >= 0.0f) return v;
    return (v * expf(64.0f - a)) * 1.60381089e-28f;  // exp(-64)
}

}  // namespace muse
