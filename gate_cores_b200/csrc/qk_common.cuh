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

// ---- Rotation-pair packing.  A 16-byte vector holds Vec<T>::N elements, i.e.
// N / 2 rotation pairs (2i, 2i + 1).  The Q/K kernel holds them as packed FP32
// pairs that group like members of two neighbouring rotation pairs: ev[j]
// holds the first members of rotation pairs 2j and 2j + 1, od[j] the second
// members.  The rotation is then elementwise on (ev, od) and costs two packed
// multiply-adds per two rotation pairs.  H = N / 4 packs of each kind.
template <typename T> struct EoPack { static constexpr int H = Vec<T>::N / 4; };

template <typename T> __device__ __forceinline__ void to_eo(const uint4& v, f32x2* ev, f32x2* od);
template <> __device__ __forceinline__ void to_eo<__nv_bfloat16>(const uint4& v, f32x2* ev, f32x2* od) {
    ev[0] = f2_make(bf16_lo(v.x), bf16_lo(v.y));
    od[0] = f2_make(bf16_hi(v.x), bf16_hi(v.y));
    ev[1] = f2_make(bf16_lo(v.z), bf16_lo(v.w));
    od[1] = f2_make(bf16_hi(v.z), bf16_hi(v.w));
}
template <> __device__ __forceinline__ void to_eo<float>(const uint4& v, f32x2* ev, f32x2* od) {
    ev[0] = f2_make(__uint_as_float(v.x), __uint_as_float(v.z));
    od[0] = f2_make(__uint_as_float(v.y), __uint_as_float(v.w));
}

// Inverse of to_eo (bf16: round to nearest even).
template <typename T> __device__ __forceinline__ uint4 from_eo(const f32x2* ev, const f32x2* od);
template <> __device__ __forceinline__ uint4 from_eo<__nv_bfloat16>(const f32x2* ev, const f32x2* od) {
    float e0, e1, e2, e3, o0, o1, o2, o3;
    f2_split(ev[0], e0, e1);
    f2_split(od[0], o0, o1);
    f2_split(ev[1], e2, e3);
    f2_split(od[1], o2, o3);
    return make_uint4(pack_bf16x2(e0, o0), pack_bf16x2(e1, o1), pack_bf16x2(e2, o2), pack_bf16x2(e3, o3));
}
template <> __device__ __forceinline__ uint4 from_eo<float>(const f32x2* ev, const f32x2* od) {
    float e0, e1, o0, o1;
    f2_split(ev[0], e0, e1);
    f2_split(od[0], o0, o1);
    return make_uint4(__float_as_uint(e0), __float_as_uint(o0), __float_as_uint(e1), __float_as_uint(o1));
}

// Rotation of normalised, cast members (e, o) of two rotation pairs by
// angles with cosines c and sines s (ns = -s):
//   FP32 rotation: e' = e c - o s, o' = e s + o c, each one product rounded and
//   one fused multiply-add (the caller casts once afterwards);
//   v2 (bf16): each product rounded to bf16, then the FP32 sum (the caller
//   casts the sum); -(o s) rounds to exactly the negated bf16 of o s.
template <typename T, bool UPCAST>
__device__ __forceinline__ void rope_eo(f32x2& e, f32x2& o, f32x2 c, f32x2 s, f32x2 ns) {
    if constexpr (UPCAST) {
        const f32x2 e2 = f2_fma(o, ns, f2_mul(e, c));
        o = f2_fma(e, s, f2_mul(o, c));
        e = e2;
    } else {
        const f32x2 e2 = f2_add(round_pair<T>(f2_mul(e, c)), round_pair<T>(f2_mul(o, ns)));
        o = f2_add(round_pair<T>(f2_mul(e, s)), round_pair<T>(f2_mul(o, c)));
        e = e2;
    }
}

// ---- bf16 pairs in one 32-bit word (low half = first element).
// Word of the low halves of w0 and w1, and of their high halves.
__device__ __forceinline__ uint32_t lo_halves(uint32_t w0, uint32_t w1) { return __byte_perm(w0, w1, 0x5410); }
__device__ __forceinline__ uint32_t hi_halves(uint32_t w0, uint32_t w1) { return __byte_perm(w0, w1, 0x7632); }
// Products and sums of bf16 pairs, each rounded once to bf16 (round to
// nearest even).  For bf16 operands they equal the FP32 operation followed
// by a cast to bf16: a product of two 8-bit significands is exact in FP32
// (for results above FP32's normal minimum), and when a sum of two bf16
// values rounds in FP32 the smaller term is below 2^-15 of the result, so
// the FP32 rounding cannot move it onto a bf16 rounding midpoint.
__device__ __forceinline__ uint32_t bf2_mul(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
__device__ __forceinline__ uint32_t bf2_add(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

}  // namespace qk
}  // namespace muse
