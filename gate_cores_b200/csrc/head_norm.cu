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
#include "qk_common.cuh"

namespace muse {
namespace {

using qk::rope_pair;
using qk::token_position;
using qk::vec_sum_sq;

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

// One CTA per tile of tokens; each warp owns one token (or, with split > 1,
// one of `split` ranges of that token's head steps).  The CTA first fills a
// shared table with cos/sin of every (token, pair) angle of the tile - one
// sincosf per pair per token - and each lane then keeps the cos/sin of its own
// VPL vectors in registers: a lane covers the same element positions of every
// head, so the values serve all heads of the token.  The token's query heads
// and then its key heads are walked in steps of RW heads, BATCH steps at a
// time with all their loads in flight; element arithmetic runs on packed FP32
// pairs and each pair is unpacked once.
template <typename T, int L, int VPL, bool ROPE, bool UPCAST, int BATCH, int MINB>
__global__ void __launch_bounds__(256, MINB) qk_norm_rope_kernel(const __grid_constant__ QkArgs a) {
    constexpr int V = Vec<T>::N;
    constexpr int P = V / 2;  // pairs per vector
    constexpr int RW = 32 / L;
    extern __shared__ float table[];  // [cos | sin][tile tokens][head_dim / 2]
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    const int split = a.split;
    const int tt = nwarps / split;  // tokens per tile
    const int sub = lane % L;
    const int slot = lane / L;
    const int nvec = a.head_dim / V;
    const int half = a.head_dim / 2;
    const float inv_width = 1.0f / (float)a.head_dim;
    const int64_t t0 = (int64_t)blockIdx.x * tt;
    const int ntok = (int)min((int64_t)tt, a.tokens - t0);
    float* cs = table;
    float* sn = table + tt * half;

    if constexpr (ROPE) {
        for (int k = warp; k < ntok; k += nwarps) {
            const float pos = (float)token_position(a, t0 + k);
            for (int p = lane; p < half; p += 32) {
                const float phi = pos * a.inv_freq[p];  // one FP32 rounding
                float sv, cv;
                sincosf(phi, &sv, &cv);
                if constexpr (!UPCAST) {
                    cv = round_to<T>(cv);
                    sv = round_to<T>(sv);
                }
                cs[k * half + p] = cv;
                sn[k * half + p] = sv;
            }
        }
        __syncthreads();
    }
    const int tok = warp / split;
    if (tok >= ntok) return;
    const int part = warp - tok * split;
    const int64_t t = t0 + tok;

    // this lane's vectors of a head: sub, sub + L, ...
    bool vok[VPL];
    uint32_t voff[VPL];
    float cv[VPL][P], sv[VPL][P];
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
        const int vi = sub + k * L;
        vok[k] = vi < nvec;
        voff[k] = (uint32_t)vi * 16u;
        if constexpr (ROPE) {
            const int tb = tok * half + (vok[k] ? vi * P : 0);
#pragma unroll
            for (int j = 0; j < P; ++j) {
                cv[k][j] = cs[tb + j];
                sv[k][j] = sn[tb + j];
            }
        }
    }
    const uint32_t head_bytes = (uint32_t)a.head_dim * sizeof(T);
    const f32x2 qs2 = f2_make(a.query_scale, a.query_scale);
    const int nst_q = (a.hq + RW - 1) / RW;
    const int nst = nst_q + (a.hkv + RW - 1) / RW;
    const int spw = (nst + split - 1) / split;
    const int g_begin = part * spw, g_end = min(nst, g_begin + spw);

    // segment 0: query heads, segment 1: key heads
#pragma unroll 1
    for (int seg = 0; seg < 2; ++seg) {
        const int s_lo = max(g_begin, seg == 0 ? 0 : nst_q) - (seg == 0 ? 0 : nst_q);
        const int s_hi = min(g_end, seg == 0 ? nst_q : nst) - (seg == 0 ? 0 : nst_q);
        if (s_lo >= s_hi) continue;
        const int count = seg == 0 ? a.hq : a.hkv;
        const bool scale = seg == 0 && a.query_scale != 1.0f;
        const char* src = seg == 0 ? static_cast<const char*>(a.q) + t * a.q_stride * (int64_t)sizeof(T)
                                   : static_cast<const char*>(a.k) + t * a.k_stride * (int64_t)sizeof(T);
        char* dst = seg == 0 ? static_cast<char*>(a.q_out) + t * a.q_out_stride * (int64_t)sizeof(T)
                             : static_cast<char*>(a.k_out) + t * a.k_out_stride * (int64_t)sizeof(T);
        for (int st0 = s_lo; st0 < s_hi; st0 += BATCH) {
            uint4 xv[BATCH][VPL];
            bool hv[BATCH];
#pragma unroll
            for (int b = 0; b < BATCH; ++b) {
                const int head = (st0 + b) * RW + slot;
                hv[b] = st0 + b < s_hi && head < count;
                const char* hs = src + (uint32_t)head * head_bytes;
#pragma unroll
                for (int k = 0; k < VPL; ++k)
                    xv[b][k] = (hv[b] && vok[k]) ? ld_stream(hs + voff[k]) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int b = 0; b < BATCH; ++b) {
                f32x2 x[VPL][P];
                f32x2 acc = f2_make(0.0f, 0.0f);
#pragma unroll
                for (int k = 0; k < VPL; ++k) {
                    to_pairs<T>(xv[b][k], x[k]);
#pragma unroll
                    for (int q = 0; q < P; ++q) acc = f2_fma(x[k][q], x[k][q], acc);
                }
                const float r = inv_rms_fast(group_sum<L>(f2_sum(acc)), inv_width, a.eps);
                const f32x2 r2 = f2_make(r, r);
                const int head = (st0 + b) * RW + slot;
                char* hd = dst + (uint32_t)head * head_bytes;
#pragma unroll
                for (int k = 0; k < VPL; ++k) {
                    f32x2 y[P];
#pragma unroll
                    for (int q = 0; q < P; ++q) {
                        f32x2 n = round_pair<T>(f2_mul(x[k][q], r2));     // cast to the Q/K dtype
                        if (scale) n = round_pair<T>(f2_mul(n, qs2));     // query_scale, cast again
                        if constexpr (ROPE) n = rope_pair<T, UPCAST>(n, cv[k][q], sv[k][q]);
                        y[q] = n;
                    }
                    if (hv[b] && vok[k]) st_vec(hd + voff[k], from_pairs<T>(y));
                }
            }
        }
    }
}

constexpr int kThreads = 256;
// Resident CTAs per SM the Q/K kernel's registers are sized for: 4 (32 warps)
// keeps enough loads in flight to cover HBM latency (measured: 2 resident
// CTAs reach about 2/3 of the copy bandwidth, 4 about 9/10).
constexpr int kQkMinBlocks = 4;

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
    constexpr int BATCH = 4;
    QkArgs a = a0;
    const int nwarps = kThreads / 32;
    const int nsteps = (a.hq + a.hkv + RW - 1) / RW;
    // Split a token's head steps over up to 8 warps while the grid would
    // leave SMs idle (decode-sized batches).
    int split = 1;
    while (split < nwarps && split < nsteps && (a.tokens * split + nwarps - 1) / nwarps < 2 * sm_count()) split *= 2;
    a.split = split;
    const int tt = nwarps / split;
    const size_t smem = ROPE ? sizeof(float) * 2 * tt * (a.head_dim / 2) : 0;
    const int64_t grid = (a.tokens + tt - 1) / tt;
    qk_norm_rope_kernel<T, L, VPL, ROPE, UPCAST, BATCH, kQkMinBlocks><<<(unsigned)grid, kThreads, smem, s>>>(a);
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
    // one 16-byte vector per lane per head (measured best at head_dim 128);
    // two for heads of more than 32 vectors
    const int nv = a.head_dim / Vec<T>::N;
    if (nv > 16) return launch_qk_modes<T, 32, 1>(use_rope, upcast, a, s);
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
