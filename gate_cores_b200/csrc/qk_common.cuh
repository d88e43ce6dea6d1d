// Device helpers of the per-head kernels (head_norm.cu).
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace muse {
namespace qk {

// Sum of squares of one 16-byte vector (two packed partial sums).
template <typename T> __device__ __forceinline__ float vec_sum_sq(const uint4& v) {
    constexpr int P = Vec<T>::N / 2;
    f32x2 p[P];
    to_pairs<T>(v, p);
    f32x2 acc = f2_mul(p[0], p[0]);
#pragma unroll
    for (int k = 1; k < P; ++k) acc = f2_fma(p[k], p[k], acc);
    return f2_sum(acc);
}

__device__ __forceinline__ int32_t token_position(const QkArgs& a, int64_t t) {
    if (a.pos_mode == 0) return __ldg(a.positions + t);
    if (a.pos_mode == 1) return (int32_t)(t % a.seqlen);
    // THD: the document d with cu[d] <= t < cu[d+1]; every index read lies in
    // [0, num_seqs - 1], whatever the array holds.
    int lo = 0, hi = a.num_seqs;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if ((int64_t)__ldg(a.cu_seqlens + mid) <= t) lo = mid; else hi = mid;
    }
    return (int32_t)(t - __ldg(a.cu_seqlens + lo));
}

// Rotation of one normalised, cast pair (a, b) by (c, s).
//   legacy / FP32 tensors: FP32 rotation (the caller casts once afterwards);
//   v2 (bf16): each product rounded to bf16, then the sum, rounded by the caller.
template <typename T, bool UPCAST>
__device__ __forceinline__ f32x2 rope_pair(f32x2 n, float c, float s) {
    float a, b;
    f2_split(n, a, b);
    if constexpr (UPCAST) {
        return f2_make(a * c - b * s, a * s + b * c);
    } else {
        const uint32_t p = pack_bf16x2(a * c, b * s);
        const uint32_t q = pack_bf16x2(a * s, b * c);
        return f2_make(bf16_lo(p) - bf16_hi(p), bf16_lo(q) + bf16_hi(q));
    }
}

}  // namespace qk
}  // namespace muse
