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

using qk::token_position;
using qk::vec_sum_sq;

// ------------------------------------------------------------ core 4 per head

// Rows of `width` elements (one head each), contiguous.  A warp handles CH
// steps of RW rows; all their loads are issued before any arithmetic.
template <typename T, int L, int VPL, int CH>
__global__ void __launch_bounds__(256) output_norm_gate_kernel(const __grid_constant__ HeadGateArgs a) {
    pdl_begin();
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
// time with all their loads in flight.  Element arithmetic runs on packed FP32
// pairs in the rotation-pair packing of to_eo (two packed multiply-adds per
// two rotations).  TAIL = false is the instance for shapes without partial
// vectors, heads or batches (every predicate drops out).
template <typename T, int L, int VPL, bool ROPE, bool UPCAST, bool TAIL, int BATCH, int MINB>
__global__ void __launch_bounds__(256, MINB) qk_norm_rope_kernel(const __grid_constant__ QkArgs a) {
    pdl_begin();
    constexpr int V = Vec<T>::N;
    constexpr int H = qk::EoPack<T>::H;
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
    const int tok = warp / split;
    const int part = warp - tok * split;
    const int64_t t = t0 + tok;
    const uint32_t head_bytes = (uint32_t)a.head_dim * sizeof(T);

    const int nst_q = (a.hq + RW - 1) / RW;
    const int nst = nst_q + (a.hkv + RW - 1) / RW;
    const int spw = (nst + split - 1) / split;
    const int g_begin = part * spw, g_end = min(nst, g_begin + spw);
    const int q_hi = min(g_end, nst_q);   // query steps [g_begin, q_hi)
    const int k_lo = max(g_begin, nst_q) - nst_q, k_hi = g_end - nst_q;  // key steps [k_lo, k_hi)
    const char* q_src = static_cast<const char*>(a.q) + t * a.q_stride * (int64_t)sizeof(T);
    const char* k_src = static_cast<const char*>(a.k) + t * a.k_stride * (int64_t)sizeof(T);

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
    if (tok >= ntok) return;

    // this lane's vectors of a head: sub, sub + L, ...; the cos / sin / -sin
    // of their rotation pairs in the packing of to_eo (8-byte table reads:
    // half and the pair offsets are even)
    bool vok[VPL];
    uint32_t voff[VPL];
    f32x2 c2[VPL][H], s2[VPL][H], n2[VPL][H];
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
        const int vi = sub + k * L;
        vok[k] = !TAIL || vi < nvec;
        voff[k] = (uint32_t)vi * 16u;
        if constexpr (ROPE) {
            const int tb = tok * half + (vok[k] ? vi * (V / 2) : 0);
#pragma unroll
            for (int j = 0; j < H; ++j) {
                c2[k][j] = *reinterpret_cast<const f32x2*>(cs + tb + 2 * j);
                s2[k][j] = *reinterpret_cast<const f32x2*>(sn + tb + 2 * j);
                n2[k][j] = f2_mul(s2[k][j], f2_make(-1.0f, -1.0f));
            }
        }
    }
    const uint32_t step_bytes = head_bytes * RW;
    const f32x2 qs2 = f2_make(a.query_scale, a.query_scale);

    // Steps [s_lo, s_hi) of one segment (the query or the key heads);
    // SCALE: multiply by query_scale and cast again after the norm's cast.
    auto run = [&](auto scale_tag, const char* seg, char* dst, int s_lo, int s_hi, int count) {
        constexpr bool SCALE = decltype(scale_tag)::value;
        const char* src = seg + (uint32_t)slot * head_bytes;
        dst += (uint32_t)slot * head_bytes;
#pragma unroll 1
        for (int st0 = s_lo; st0 < s_hi; st0 += BATCH) {
            uint4 xv[BATCH][VPL];
            bool hv[BATCH];
#pragma unroll
            for (int b = 0; b < BATCH; ++b) {
                hv[b] = !TAIL || (st0 + b < s_hi && (st0 + b) * RW + slot < count);
                const char* hs = src + (uint32_t)(st0 + b) * step_bytes;
#pragma unroll
                for (int k = 0; k < VPL; ++k)
                    xv[b][k] = (hv[b] && vok[k]) ? ld_stream(hs + voff[k]) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int b = 0; b < BATCH; ++b) {
                f32x2 e[VPL][H], o[VPL][H];
                f32x2 acc = f2_make(0.0f, 0.0f);
#pragma unroll
                for (int k = 0; k < VPL; ++k) {
                    qk::to_eo<T>(xv[b][k], e[k], o[k]);
#pragma unroll
                    for (int j = 0; j < H; ++j) {
                        acc = f2_fma(e[k][j], e[k][j], acc);
                        acc = f2_fma(o[k][j], o[k][j], acc);
                    }
                }
                const float r = inv_rms_fast(group_sum<L>(f2_sum(acc)), inv_width, a.eps);
                const f32x2 r2 = f2_make(r, r);
                char* hd = dst + (uint32_t)(st0 + b) * step_bytes;
#pragma unroll
                for (int k = 0; k < VPL; ++k) {
#pragma unroll
                    for (int j = 0; j < H; ++j) {
                        f32x2 ev = round_pair<T>(f2_mul(e[k][j], r2));  // cast to the Q/K dtype
                        f32x2 ov = round_pair<T>(f2_mul(o[k][j], r2));
                        if constexpr (SCALE) {                         // query_scale, cast again
                            ev = round_pair<T>(f2_mul(ev, qs2));
                            ov = round_pair<T>(f2_mul(ov, qs2));
                        }
                        if constexpr (ROPE) qk::rope_eo<T, UPCAST>(ev, ov, c2[k][j], s2[k][j], n2[k][j]);
                        e[k][j] = ev;
                        o[k][j] = ov;
                    }
                    if (hv[b] && vok[k]) st_vec(hd + voff[k], qk::from_eo<T>(e[k], o[k]));
                }
            }
        }
    };

    if (g_begin < q_hi) {
        char* dst = static_cast<char*>(a.q_out) + t * a.q_out_stride * (int64_t)sizeof(T);
        if (a.query_scale != 1.0f)
            run(std::true_type{}, q_src, dst, g_begin, q_hi, a.hq);
        else
            run(std::false_type{}, q_src, dst, g_begin, q_hi, a.hq);
    }
    if (k_lo < k_hi) {
        char* dst = static_cast<char*>(a.k_out) + t * a.k_out_stride * (int64_t)sizeof(T);
        run(std::false_type{}, k_src, dst, k_lo, k_hi, a.hkv);
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
    return launch_pdl(output_norm_gate_kernel<T, L, VPL, CH>, (unsigned)grid, kThreads, 0, s, a);
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
    const int nst_q = (a.hq + RW - 1) / RW, nst_k = (a.hkv + RW - 1) / RW;
    // Split a token's head steps over up to 8 warps while the grid would
    // leave SMs idle (decode-sized batches).
    int split = 1;
    while (split < nwarps && split < nst_q + nst_k &&
           (a.tokens * split + nwarps - 1) / nwarps < 2 * sm_count())
        split *= 2;
    a.split = split;
    const int tt = nwarps / split;
    const size_t smem = ROPE ? sizeof(float) * 2 * tt * (a.head_dim / 2) : 0;
    const int64_t grid = (a.tokens + tt - 1) / tt;
    const bool exact = split == 1 && a.head_dim / Vec<T>::N == L * VPL && a.hq % RW == 0 &&
                       a.hkv % RW == 0 && nst_q % BATCH == 0 && nst_k % BATCH == 0;
    if (exact)
        return launch_pdl(qk_norm_rope_kernel<T, L, VPL, ROPE, UPCAST, false, BATCH, kQkMinBlocks>,
                          (unsigned)grid, kThreads, smem, s, a);
    return launch_pdl(qk_norm_rope_kernel<T, L, VPL, ROPE, UPCAST, true, BATCH, kQkMinBlocks>,
                      (unsigned)grid, kThreads, smem, s, a);
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
