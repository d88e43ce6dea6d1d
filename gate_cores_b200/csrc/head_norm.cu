// Per-head kernels: core 3 (Q/K norm + RoPE) and core 4 with one norm per
// head.  A head of D elements is NV = D / Vec<T>::N 16-byte vectors; each lane
// owns VPL of them (vectors sub, sub + L, ...: every load instruction of a
// warp reads whole 32-byte sectors), so L = NV / VPL lanes (rounded up to a
// power of two) cover a head and a warp covers RW = 32 / L heads per step.
// The per-head sum of squares is a butterfly over the L lanes; no CTA barrier
// except the one after core 3's cos/sin table.  Both grids are one-shot: each
// CTA handles one tile of work and exits.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace muse {
namespace {

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

// ------------------------------------------------------------ core 4 per head

// Rows of `width` elements (one head each), contiguous.  A warp handles CH
// steps of RW rows; all their loads are issued before any arithmetic.
template <typename T, int L, int VPL, int CH>
__global__ void __launch_bounds__(256) output_norm_gate_kernel(const __grid_constant__ HeadGateArgs a) {
    constexpr int V = Vec<T>::N;
    constexpr int RW = 32 / L;
    const int lane = threadIdx.x & 31;
    const int sub = lane % L;
    const int slot = lane / L;
    const int nvec = a.width / V;
    const float inv_width = 1.0f / (float)a.width;
    const int64_t row_bytes = (int64_t)a.width * sizeof(T);
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t base = warp * (CH * RW);

    uint4 ov[CH][VPL], gv[CH][VPL];
    bool ok[CH][VPL];
#pragma unroll
    for (int c = 0; c < CH; ++c) {
        const int64_t row = base + c * RW + slot;
#pragma unroll
        for (int k = 0; k < VPL; ++k) {
            const int vi = sub + k * L;
            ok[c][k] = vi < nvec && row < a.rows;
            const int64_t off = row * row_bytes + (int64_t)vi * 16;
            ov[c][k] = ok[c][k] ? ld_stream(static_cast<const char*>(a.o) + off) : make_uint4(0, 0, 0, 0);
            gv[c][k] = ok[c][k] ? ld_stream(static_cast<const char*>(a.gate) + off) : make_uint4(0, 0, 0, 0);
        }
    }
#pragma unroll
    for (int c = 0; c < CH; ++c) {
        float ss = 0.0f;
#pragma unroll
        for (int k = 0; k < VPL; ++k) ss += vec_sum_sq<T>(ov[c][k]);
        const float r = inv_rms_fast(group_sum<L>(ss), inv_width, a.eps);
        const int64_t row = base + c * RW + slot;
#pragma unroll
        for (int k = 0; k < VPL; ++k) {
            float of[V], gf[V], y[V];
            unpack<T>(ov[c][k], of);
            unpack<T>(gv[c][k], gf);
#pragma unroll
            for (int e = 0; e < V; ++e) y[e] = times_sigmoid<T>(of[e] * r, gf[e]);
            if (ok[c][k])
                st_vec(static_cast<char*>(a.y) + row * row_bytes + (int64_t)(sub + k * L) * 16, pack<T>(y));
        }
    }
}

// ------------------------------------------------------------------ core 3

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

// Normalised, cast, optionally scaled and rotated 16-byte vector of one head.
// cs/sn: cos/sin of this vector's Vec<T>::N / 2 pairs.
template <typename T, bool ROPE, bool UPCAST>
__device__ __forceinline__ uint4 qk_vec(const uint4& in, float r, bool scale, float qs,
                                        const float* cs, const float* sn);

template <bool ROPE, bool UPCAST>
__device__ __forceinline__ uint32_t qk_pair_bf16(uint32_t w, f32x2 r2, bool scale, float qs, float c, float s) {
    // cast of the normalised pair to bf16 (cvt.rn.bf16x2)
    float n0, n1;
    f2_split(f2_mul(f2_make(bf16_lo(w), bf16_hi(w)), r2), n0, n1);
    uint32_t n = pack_bf16x2(n0, n1);
    if (scale) n = pack_bf16x2(bf16_lo(n) * qs, bf16_hi(n) * qs);
    if constexpr (!ROPE) {
        return n;
    } else {
        const float x0 = bf16_lo(n), x1 = bf16_hi(n);
        if constexpr (UPCAST) {
            return pack_bf16x2(x0 * c - x1 * s, x0 * s + x1 * c);
        } else {
            // v2: each product rounded to bf16 before the sum, the sum cast again
            const uint32_t p = pack_bf16x2(x0 * c, x1 * s);
            const uint32_t q = pack_bf16x2(x0 * s, x1 * c);
            return pack_bf16x2(bf16_lo(p) - bf16_hi(p), bf16_lo(q) + bf16_hi(q));
        }
    }
}

template <>
__device__ __forceinline__ uint4 qk_vec<__nv_bfloat16, false, true>(const uint4& in, float r, bool scale, float qs,
                                                                   const float*, const float*) {
    const f32x2 r2 = f2_make(r, r);
    return make_uint4(qk_pair_bf16<false, true>(in.x, r2, scale, qs, 0, 0),
                      qk_pair_bf16<false, true>(in.y, r2, scale, qs, 0, 0),
                      qk_pair_bf16<false, true>(in.z, r2, scale, qs, 0, 0),
                      qk_pair_bf16<false, true>(in.w, r2, scale, qs, 0, 0));
}
template <>
__device__ __forceinline__ uint4 qk_vec<__nv_bfloat16, true, true>(const uint4& in, float r, bool scale, float qs,
                                                                  const float* c, const float* s) {
    const f32x2 r2 = f2_make(r, r);
    return make_uint4(qk_pair_bf16<true, true>(in.x, r2, scale, qs, c[0], s[0]),
                      qk_pair_bf16<true, true>(in.y, r2, scale, qs, c[1], s[1]),
                      qk_pair_bf16<true, true>(in.z, r2, scale, qs, c[2], s[2]),
                      qk_pair_bf16<true, true>(in.w, r2, scale, qs, c[3], s[3]));
}
template <>
__device__ __forceinline__ uint4 qk_vec<__nv_bfloat16, true, false>(const uint4& in, float r, bool scale, float qs,
                                                                   const float* c, const float* s) {
    const f32x2 r2 = f2_make(r, r);
    return make_uint4(qk_pair_bf16<true, false>(in.x, r2, scale, qs, c[0], s[0]),
                      qk_pair_bf16<true, false>(in.y, r2, scale, qs, c[1], s[1]),
                      qk_pair_bf16<true, false>(in.z, r2, scale, qs, c[2], s[2]),
                      qk_pair_bf16<true, false>(in.w, r2, scale, qs, c[3], s[3]));
}
// FP32 tensors: the casts are exact and the rotation is FP32 in both modes.
template <bool ROPE>
__device__ __forceinline__ uint4 qk_vec_f32(const uint4& in, float r, bool scale, float qs,
                                            const float* c, const float* s) {
    float f[4];
    unpack<float>(in, f);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        f[e] = f[e] * r;
        if (scale) f[e] = f[e] * qs;
    }
    if constexpr (ROPE) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const float x0 = f[2 * j], x1 = f[2 * j + 1];
            f[2 * j] = x0 * c[j] - x1 * s[j];
            f[2 * j + 1] = x0 * s[j] + x1 * c[j];
        }
    }
    return pack<float>(f);
}
template <>
__device__ __forceinline__ uint4 qk_vec<float, false, true>(const uint4& in, float r, bool scale, float qs,
                                                           const float* c, const float* s) {
    return qk_vec_f32<false>(in, r, scale, qs, c, s);
}
template <>
__device__ __forceinline__ uint4 qk_vec<float, true, true>(const uint4& in, float r, bool scale, float qs,
                                                          const float* c, const float* s) {
    return qk_vec_f32<true>(in, r, scale, qs, c, s);
}

// One CTA per tile of tile_tokens consecutive tokens.  The CTA first fills a
// shared table with cos/sin of every (token, pair) angle - one sincosf per pair
// per token - then its warps walk the tile's (token, head step) units, CH
// units at a time with all their loads in flight.  Head steps cover query
// heads first, then key heads.
template <typename T, int L, int VPL, bool ROPE, bool UPCAST, int CH>
__global__ void __launch_bounds__(256) qk_norm_rope_kernel(const __grid_constant__ QkArgs a) {
    constexpr int V = Vec<T>::N;
    constexpr int P = V / 2;  // rotation pairs per vector
    constexpr int RW = 32 / L;
    extern __shared__ float table[];  // [cos | sin][tile_tokens][head_dim / 2]
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    const int sub = lane % L;
    const int slot = lane / L;
    const int nvec = a.head_dim / V;
    const float inv_width = 1.0f / (float)a.head_dim;
    const int half = a.head_dim / 2;
    const int tt = a.tile_tokens;
    const int nh = a.hq + a.hkv;
    const int nsteps = (nh + RW - 1) / RW;
    const bool scale_q = a.query_scale != 1.0f;
    const int64_t t0 = (int64_t)blockIdx.x * tt;
    const int ntok = (int)min((int64_t)tt, a.tokens - t0);
    float* cs = table;
    float* sn = table + tt * half;

    if constexpr (ROPE) {
        for (int i = threadIdx.x; i < ntok * half; i += blockDim.x) {
            const int k = i / half;
            const float pos = (float)token_position(a, t0 + k);
            const float phi = pos * a.inv_freq[i - k * half];  // one FP32 rounding
            float sv, cv;
            sincosf(phi, &sv, &cv);
            if constexpr (!UPCAST) {
                cv = round_to<T>(cv);
                sv = round_to<T>(sv);
            }
            cs[i] = cv;
            sn[i] = sv;
        }
        __syncthreads();
    }
    const int units = ntok * nsteps;
    for (int u0 = warp * CH; u0 < units; u0 += nwarps * CH) {
        uint4 xv[CH][VPL];
        int tok[CH], head[CH];
        bool ok[CH][VPL];
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            const int u = u0 + c;
            tok[c] = u / nsteps;
            head[c] = (u - tok[c] * nsteps) * RW + slot;
            const bool hv = u < units && head[c] < nh;
            const int64_t t = t0 + tok[c];
            const char* src = head[c] < a.hq
                ? static_cast<const char*>(a.q) + (t * a.q_stride + (int64_t)head[c] * a.head_dim) * (int64_t)sizeof(T)
                : static_cast<const char*>(a.k) + (t * a.k_stride + (int64_t)(head[c] - a.hq) * a.head_dim) * (int64_t)sizeof(T);
#pragma unroll
            for (int k = 0; k < VPL; ++k) {
                const int vi = sub + k * L;
                ok[c][k] = hv && vi < nvec;
                xv[c][k] = ok[c][k] ? ld_stream(src + (int64_t)vi * 16) : make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            float ss = 0.0f;
#pragma unroll
            for (int k = 0; k < VPL; ++k) ss += vec_sum_sq<T>(xv[c][k]);
            const float r = inv_rms_fast(group_sum<L>(ss), inv_width, a.eps);
            const bool is_q = head[c] < a.hq;
            const int64_t t = t0 + tok[c];
            char* dst = is_q
                ? static_cast<char*>(a.q_out) + (t * a.q_out_stride + (int64_t)head[c] * a.head_dim) * (int64_t)sizeof(T)
                : static_cast<char*>(a.k_out) + (t * a.k_out_stride + (int64_t)(head[c] - a.hq) * a.head_dim) * (int64_t)sizeof(T);
#pragma unroll
            for (int k = 0; k < VPL; ++k) {
                const int vi = sub + k * L;
                // this vector's cos/sin (table row 0 for idle lanes and units)
                const int tb = ok[c][k] ? tok[c] * half + vi * P : 0;
                float cv[P], sv[P];
                if constexpr (ROPE) {
#pragma unroll
                    for (int j = 0; j < P; ++j) {
                        cv[j] = cs[tb + j];
                        sv[j] = sn[tb + j];
                    }
                }
                const uint4 y = qk_vec<T, ROPE, UPCAST>(xv[c][k], r, is_q && scale_q, a.query_scale, cv, sv);
                if (ok[c][k]) st_vec(dst + (int64_t)vi * 16, y);
            }
        }
    }
}

int gcd(int x, int y) { return y == 0 ? x : gcd(y, x % y); }

constexpr int kThreads = 256;

template <typename T, int L, int VPL, int CH>
cudaError_t launch_head_gate_l(const HeadGateArgs& a, cudaStream_t s) {
    constexpr int RW = 32 / L;
    const int64_t rows_per_cta = (int64_t)(kThreads / 32) * CH * RW;
    const int64_t grid = (a.rows + rows_per_cta - 1) / rows_per_cta;
    output_norm_gate_kernel<T, L, VPL, CH><<<(unsigned)grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

// Lanes per head: NV / VPL rounded up to a power of two; two vectors per lane
// when a head has at least 16.
template <typename T>
cudaError_t launch_head_gate_t(const HeadGateArgs& a, cudaStream_t s) {
    const int nv = a.width / Vec<T>::N;
    if (nv >= 16) {
        const int lanes = (nv + 1) / 2;
        if (lanes <= 8) return launch_head_gate_l<T, 8, 2, 1>(a, s);
        if (lanes <= 16) return launch_head_gate_l<T, 16, 2, 1>(a, s);
        return launch_head_gate_l<T, 32, 2, 1>(a, s);
    }
    if (nv <= 1) return launch_head_gate_l<T, 1, 1, 2>(a, s);
    if (nv <= 2) return launch_head_gate_l<T, 2, 1, 2>(a, s);
    if (nv <= 4) return launch_head_gate_l<T, 4, 1, 2>(a, s);
    if (nv <= 8) return launch_head_gate_l<T, 8, 1, 2>(a, s);
    return launch_head_gate_l<T, 16, 1, 2>(a, s);
}

template <typename T, int L, int VPL, bool ROPE, bool UPCAST>
cudaError_t launch_qk_l(const QkArgs& a0, cudaStream_t s) {
    constexpr int RW = 32 / L;
    constexpr int CH = 2;
    QkArgs a = a0;
    const int nsteps = (a.hq + a.hkv + RW - 1) / RW;
    // Tile: enough tokens that the tile's units fill every warp's CH-unit
    // rounds exactly, shrunk while the grid would leave SMs without a CTA.
    const int per_round = (kThreads / 32) * CH;
    int tt = per_round / gcd(nsteps, per_round);
    if (tt > kMaxTileTokens) tt = kMaxTileTokens;
    while (tt > 1 && (a.tokens + tt - 1) / tt < 2 * sm_count()) tt /= 2;
    a.tile_tokens = tt;
    const size_t smem = ROPE ? sizeof(float) * 2 * tt * (a.head_dim / 2) : 0;
    const int64_t grid = (a.tokens + tt - 1) / tt;
    qk_norm_rope_kernel<T, L, VPL, ROPE, UPCAST, CH><<<(unsigned)grid, kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

template <typename T, int L, int VPL>
cudaError_t launch_qk_modes(int use_rope, int upcast, const QkArgs& a, cudaStream_t s) {
    if (!use_rope) return launch_qk_l<T, L, VPL, false, true>(a, s);
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        if (!upcast) return launch_qk_l<T, L, VPL, true, false>(a, s);
    }
    return launch_qk_l<T, L, VPL, true, true>(a, s);
}

template <typename T>
cudaError_t launch_qk_t(int use_rope, int upcast, const QkArgs& a, cudaStream_t s) {
    const int nv = a.head_dim / Vec<T>::N;
    if (nv >= 16) {
        const int lanes = (nv + 1) / 2;
        if (lanes <= 8) return launch_qk_modes<T, 8, 2>(use_rope, upcast, a, s);
        if (lanes <= 16) return launch_qk_modes<T, 16, 2>(use_rope, upcast, a, s);
        return launch_qk_modes<T, 32, 2>(use_rope, upcast, a, s);
    }
    if (nv <= 1) return launch_qk_modes<T, 1, 1>(use_rope, upcast, a, s);
    if (nv <= 2) return launch_qk_modes<T, 2, 1>(use_rope, upcast, a, s);
    if (nv <= 4) return launch_qk_modes<T, 4, 1>(use_rope, upcast, a, s);
    if (nv <= 8) return launch_qk_modes<T, 8, 1>(use_rope, upcast, a, s);
    return launch_qk_modes<T, 16, 1>(use_rope, upcast, a, s);
}

}  // namespace

cudaError_t launch_head_gate(int dtype, const HeadGateArgs& a, cudaStream_t s) {
    return dtype == 0 ? launch_head_gate_t<__nv_bfloat16>(a, s) : launch_head_gate_t<float>(a, s);
}

cudaError_t launch_qk(int dtype, int use_rope, int upcast_rope, const QkArgs& a, cudaStream_t s) {
    // FP32 tensors rotate in FP32 in both modes.
    if (dtype != 0) return launch_qk_t<float>(use_rope, 1, a, s);
    return launch_qk_t<__nv_bfloat16>(use_rope, upcast_rope, a, s);
}

}  // namespace muse
