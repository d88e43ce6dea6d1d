// Backward of the per-head cores: core 4 (_output_norm_gate_core) and core 3
// (_qk_norm_rope_core, FP32 or v2 rotation).  Derivatives of the forward maps,
// evaluated in FP32 from the saved forward inputs, with every dtype boundary
// the forward materialises rounding the gradient that flows back through it:
//
//   core 4, per group of G elements (a head, or a whole token):
//     s = sigmoid(g), n = o r(o);  dn = dy s;
//     do = r dn - r^3 o (sum_j dn_j o_j) / G;   dg = dy n s (1 - s)
//   core 3, per head of D elements:
//     dm = R(phi)^T dy  (da = c dy0 + s dy1, db = -s dy0 + c dy1, FP32);
//     dn = cast(dm);  query heads: dn = cast(dn * query_scale);
//     dx = r dn - r^3 x (sum_j dn_j x_j) / D
//   v2 rotation (bf16; C, S the bf16 cos and sin): the forward's bf16
//   products and sums give dn = (cast(cast(dy0 C) + cast(dy1 S)),
//   cast(cast(dy1 C) - cast(dy0 S))) per pair before the query scaling.
//
// Layouts, lanes per head and the Q/K ring (each warp streams its batches of
// head steps through its own shared-memory slots with cp.async.bulk, here two
// tensors per batch: the forward input and the incoming gradient) follow the
// forward kernels in head_norm.cu.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "qk_common.cuh"

namespace muse {
namespace {
__device__ unsigned int g_device_error;  // nonzero: an mbarrier wait of the Q/K backward ring timed out
}  // namespace
}  // namespace muse

#include "tma_pipe.cuh"

namespace muse {
namespace {

using qk::token_position;

// sigmoid(g) and its slope sigmoid'(g) = e^-|g| / (1 + e^-|g|)^2, the slope
// as sp * slope_scale<T>() with the power of two applied last: for bf16
// outputs t' = 2^64 e^-|g| stays normal for |g| < 132, so a gradient that
// ends in the bf16 subnormal range is rounded once.  FP32 outputs use expf and
// IEEE division (beyond |g| = 80 via e^-|g| = e^(64-|g|) e^-64).
template <typename T> __host__ __device__ constexpr float slope_scale() {
    return std::is_same<T, float>::value ? 1.0f : 0x1p-64f;
}
template <typename T> __device__ __forceinline__ void sigmoid_slope(float g, float& s, float& sp);
template <> __device__ __forceinline__ void sigmoid_slope<__nv_bfloat16>(float g, float& s, float& sp) {
    const float a = fabsf(g);
    const float tp = exp2_approx(fmaf(-a, 1.44269504088896341f, 64.0f));
    const float d = rcp_approx_ftz(fmaf(tp, 0x1p-64f, 1.0f));  // 1 / (1 + e^-|g|), argument in [1, 2]
    s = g >= 0.0f ? d : (tp * d) * 0x1p-64f;
    sp = (tp * d) * d;
}
template <> __device__ __forceinline__ void sigmoid_slope<float>(float g, float& s, float& sp) {
    const float a = fabsf(g);
    if (a <= 80.0f) {
        const float t = expf(-a);
        const float d = 1.0f / (1.0f + t);
        s = g >= 0.0f ? d : t * d;
        sp = (t * d) * d;
    } else {
        const float t = expf(64.0f - a) * 1.60381089e-28f;  // e^-64; 1 + e^-|g| rounds to 1
        s = g >= 0.0f ? 1.0f : t;
        sp = t;
    }
}

// ------------------------------------------------------ core 4, per head

// Groups of `width` elements, L lanes x VPL 16-byte vectors per group, RW =
// 32 / L groups per warp; one-shot grid.
template <typename T, int L, int VPL>
__global__ void __launch_bounds__(256) output_norm_gate_bwd_kernel(const __grid_constant__ GateBwdArgs a) {
    pdl_begin();
    constexpr int V = Vec<T>::N;
    constexpr int RW = 32 / L;
    const int lane = threadIdx.x & 31;
    const int sub = lane % L;
    const int slot = lane / L;
    const int nvec = a.width / V;
    const float inv_width = 1.0f / (float)a.width;
    const int64_t row_bytes = (int64_t)a.width * sizeof(T);
    const int64_t row = (((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5) * RW + slot;

    uint4 ov[VPL], gv[VPL], dv[VPL];
    bool ok[VPL];
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
        const int vi = sub + k * L;
        ok[k] = vi < nvec && row < a.rows;
        const int64_t off = row * row_bytes + (int64_t)vi * 16;
        ov[k] = ok[k] ? ld_stream(static_cast<const char*>(a.o) + off) : make_uint4(0, 0, 0, 0);
        gv[k] = ok[k] ? ld_stream(static_cast<const char*>(a.gate) + off) : make_uint4(0, 0, 0, 0);
        dv[k] = ok[k] ? ld_stream(static_cast<const char*>(a.dy) + off) : make_uint4(0, 0, 0, 0);
    }
    float of[VPL][V], dn[VPL][V], dyf[VPL][V], sp[VPL][V];
    float ss = 0.0f, cd = 0.0f;
    constexpr float scale = slope_scale<T>();
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
        float gf[V];
        unpack<T>(ov[k], of[k]);
        unpack<T>(gv[k], gf);
        unpack<T>(dv[k], dyf[k]);
#pragma unroll
        for (int e = 0; e < V; ++e) {
            float s;
            sigmoid_slope<T>(gf[e], s, sp[k][e]);
            dn[k][e] = dyf[k][e] * s;
            ss = fmaf(of[k][e], of[k][e], ss);
            cd = fmaf(dn[k][e], of[k][e], cd);
        }
    }
    ss = group_sum<L>(ss);
    cd = group_sum<L>(cd);
    const float r = inv_rms_fast(ss, inv_width, a.eps);
    const float cr = r * r * r * cd * inv_width;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
        float dof[V], dgf[V];
#pragma unroll
        for (int e = 0; e < V; ++e) {
            dof[e] = r * dn[k][e] - cr * of[k][e];
            dgf[e] = ((dyf[k][e] * (of[k][e] * r)) * sp[k][e]) * scale;
        }
        if (ok[k]) {
            const int64_t off = row * row_bytes + (int64_t)(sub + k * L) * 16;
            st_vec(static_cast<char*>(a.d_o) + off, pack<T>(dof));
            st_vec(static_cast<char*>(a.dgate) + off, pack<T>(dgf));
        }
    }
}

// ------------------------------------------------ core 4, one group per CTA

// Wide groups (a whole token): one CTA per group, VPT vectors per thread,
// the two sums reduced through shared memory.
template <typename T, int VPT>
__global__ void __launch_bounds__(512) output_norm_gate_group_bwd_kernel(const __grid_constant__ GateBwdArgs a) {
    pdl_begin();
    constexpr int V = Vec<T>::N;
    __shared__ float red[2][32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const int nvec = a.width / V;
    const float inv_width = 1.0f / (float)a.width;
    const int64_t base = (int64_t)blockIdx.x * a.width * sizeof(T);
    uint4 ov[VPT], gv[VPT], dv[VPT];
    bool ok[VPT];
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
        const int vi = tid + k * blockDim.x;
        ok[k] = vi < nvec;
        const int64_t off = base + (int64_t)vi * 16;
        ov[k] = ok[k] ? ld_stream(static_cast<const char*>(a.o) + off) : make_uint4(0, 0, 0, 0);
        gv[k] = ok[k] ? ld_stream(static_cast<const char*>(a.gate) + off) : make_uint4(0, 0, 0, 0);
        dv[k] = ok[k] ? ld_stream(static_cast<const char*>(a.dy) + off) : make_uint4(0, 0, 0, 0);
    }
    float of[VPT][V], dn[VPT][V], dyf[VPT][V], sp[VPT][V];
    float ss = 0.0f, cd = 0.0f;
    constexpr float scale = slope_scale<T>();
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
        float gf[V];
        unpack<T>(ov[k], of[k]);
        unpack<T>(gv[k], gf);
        unpack<T>(dv[k], dyf[k]);
#pragma unroll
        for (int e = 0; e < V; ++e) {
            float s;
            sigmoid_slope<T>(gf[e], s, sp[k][e]);
            dn[k][e] = dyf[k][e] * s;
            ss = fmaf(of[k][e], of[k][e], ss);
            cd = fmaf(dn[k][e], of[k][e], cd);
        }
    }
    ss = group_sum<32>(ss);
    cd = group_sum<32>(cd);
    if (lane == 0) {
        red[0][warp] = ss;
        red[1][warp] = cd;
    }
    __syncthreads();
    ss = group_sum<32>(lane < nw ? red[0][lane] : 0.0f);
    cd = group_sum<32>(lane < nw ? red[1][lane] : 0.0f);
    const float r = inv_rms_fast(ss, inv_width, a.eps);
    const float cr = r * r * r * cd * inv_width;
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
        float dof[V], dgf[V];
#pragma unroll
        for (int e = 0; e < V; ++e) {
            dof[e] = r * dn[k][e] - cr * of[k][e];
            dgf[e] = ((dyf[k][e] * (of[k][e] * r)) * sp[k][e]) * scale;
        }
        if (ok[k]) {
            const int64_t off = base + (int64_t)(tid + k * blockDim.x) * 16;
            st_vec(static_cast<char*>(a.d_o) + off, pack<T>(dof));
            st_vec(static_cast<char*>(a.dgate) + off, pack<T>(dgf));
        }
    }
}

// ------------------------------------------------------------ core 3

// A persistent grid whose warps split the tokens x batches units evenly in
// token order (a unit: BATCH head steps of the forward input and of the
// incoming gradient, both brought into one slot of the warp's ring of R by two
// bulk copies on one mbarrier; a warp takes a contiguous range of units, so
// every warp streams the same amount to within one unit); each lane computes
// the cos / sin of its own rotation pairs when its warp reaches a new token.
// Measured on B200 at prefill sizes against one-shot CTAs of whole-token work
// (2.3 waves of 8192 tokens on 3552 warp slots): 7% faster back to back, 13%
// alone; units dealt round-robin instead (angles recomputed per unit) were as
// slow as the one-shot grid.
template <typename T, int L, bool ROPE, bool V2, bool TAIL, int BATCH, int R>
__global__ void __launch_bounds__(256, 3) qk_norm_rope_bwd_kernel(const __grid_constant__ QkBwdArgs A) {
    pdl_begin();
    const QkArgs& a = A.f;
    constexpr int V = Vec<T>::N;
    constexpr int H = qk::EoPack<T>::H;
    constexpr int RW = 32 / L;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t bars[8][R];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int sub = lane % L;
    const int slot = lane / L;
    const int nvec = a.head_dim / V;
    const float inv_width = 1.0f / (float)a.head_dim;
    const uint32_t head_bytes = (uint32_t)a.head_dim * sizeof(T);
    const uint32_t half_slot = (BATCH * RW * head_bytes + 127u) & ~127u;
    const uint32_t slot_bytes = 2 * half_slot;
    unsigned char* ring = smem_raw + (uint32_t)warp * R * slot_bytes;

    const int nst_q = (a.hq + RW - 1) / RW, nst_k = (a.hkv + RW - 1) / RW;
    const int nbq = (nst_q + BATCH - 1) / BATCH;
    const int nb = nbq + (nst_k + BATCH - 1) / BATCH;
    const int64_t nw = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t gw = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp;
    const int64_t units = a.tokens * nb;
    const int64_t u0 = gw * units / nw;
    const int n = (int)((gw + 1) * units / nw - u0);
    if (n <= 0) return;

    auto batch = [&](int j, int& st0, int& s_hi, int& count, bool& isq) {
        isq = j < nbq;
        st0 = isq ? j * BATCH : (j - nbq) * BATCH;
        s_hi = isq ? nst_q : nst_k;
        count = isq ? a.hq : a.hkv;
    };
    int64_t it = u0 / nb;
    int ij = (int)(u0 - it * nb);
    auto issue = [&](int i) {
        int st0, s_hi, count;
        bool isq;
        batch(ij, st0, s_hi, count, isq);
        const int h0 = st0 * RW, h1 = min(count, min(st0 + BATCH, s_hi) * RW);
        const uint32_t bytes = (uint32_t)(h1 - h0) * head_bytes;
        const char* xs = isq ? static_cast<const char*>(a.q) + it * a.q_stride * (int64_t)sizeof(T)
                             : static_cast<const char*>(a.k) + it * a.k_stride * (int64_t)sizeof(T);
        const char* gs = isq ? static_cast<const char*>(A.gq) + it * A.gq_stride * (int64_t)sizeof(T)
                             : static_cast<const char*>(A.gk) + it * A.gk_stride * (int64_t)sizeof(T);
        uint64_t* bar = &bars[warp][i % R];
        unsigned char* dst = ring + (i % R) * slot_bytes;
        pipe::mbar_arrive_expect_tx(bar, 2 * bytes);
        pipe::bulk_g2s(dst, xs + (uint32_t)h0 * head_bytes, bytes, bar);
        pipe::bulk_g2s(dst + half_slot, gs + (uint32_t)h0 * head_bytes, bytes, bar);
        if (++ij == nb) {
            ij = 0;
            ++it;
        }
    };
    int issued = 0;
    if (lane == 0) {
        for (int r = 0; r < R; ++r) pipe::mbar_init(&bars[warp][r], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (; issued < min(R, n); ++issued) issue(issued);
    }
    __syncwarp();

    const bool vok = !TAIL || sub < nvec;
    const uint32_t voff = (uint32_t)sub * 16u;
    // v2 with bf16 Q/K: the rounded cos / sin also as bf16 pairs
    constexpr bool BF2 = ROPE && V2 && std::is_same<T, __nv_bfloat16>::value;
    f32x2 c2[H], s2[H], n2[H];
    uint32_t cb[BF2 ? H : 1], sb[BF2 ? H : 1], nb2[BF2 ? H : 1];
    auto set_angles = [&](int64_t t) {
        if constexpr (ROPE) {
            const float pos = (float)token_position(a, t);
            const int p0 = (vok ? sub : 0) * (V / 2);
#pragma unroll
            for (int j = 0; j < H; ++j) {
                float s0, c0, s1, c1;
                sincosf(pos * a.inv_freq[p0 + 2 * j], &s0, &c0);  // one FP32 rounding of the angle
                sincosf(pos * a.inv_freq[p0 + 2 * j + 1], &s1, &c1);
                if constexpr (V2) {
                    c0 = round_to<T>(c0);
                    s0 = round_to<T>(s0);
                    c1 = round_to<T>(c1);
                    s1 = round_to<T>(s1);
                }
                c2[j] = f2_make(c0, c1);
                s2[j] = f2_make(s0, s1);
                n2[j] = f2_make(-s0, -s1);
                if constexpr (BF2) {  // exact: the values are bf16 already
                    cb[j] = pack_bf16x2(c0, c1);
                    sb[j] = pack_bf16x2(s0, s1);
                    nb2[j] = pack_bf16x2(-s0, -s1);
                }
            }
        }
    };
    const f32x2 qs2 = f2_make(a.query_scale, a.query_scale);
    const bool scaled = a.query_scale != 1.0f;
    auto compute = [&](auto scale_tag, const uint4 (&xv)[BATCH], const uint4 (&gv)[BATCH],
                       const bool (&hv)[BATCH], char* dst) {
        constexpr bool SCALE = decltype(scale_tag)::value;
#pragma unroll
        for (int b = 0; b < BATCH; ++b) {
            f32x2 xe[H], xo[H], de[H], dd[H];
            qk::to_eo<T>(xv[b], xe, xo);
            if constexpr (!BF2) qk::to_eo<T>(gv[b], de, dd);
            f32x2 ss = f2_make(0.0f, 0.0f), cd = f2_make(0.0f, 0.0f);
#pragma unroll
            for (int j = 0; j < H; ++j) {
                f32x2 me, mo;
                if constexpr (BF2) {
                    // v2, bf16 Q/K: the same bf16 products and sums as below on
                    // bf16 pairs (first and second members of rotation pairs
                    // 2j, 2j + 1 of the incoming gradient), already bf16
                    static_assert(H == 2, "a 16-byte vector holds 4 rotation pairs of bf16");
                    const uint32_t w0 = j == 0 ? gv[b].x : gv[b].z, w1 = j == 0 ? gv[b].y : gv[b].w;
                    const uint32_t e = qk::lo_halves(w0, w1), o = qk::hi_halves(w0, w1);
                    const uint32_t me_b = qk::bf2_add(qk::bf2_mul(e, cb[j]), qk::bf2_mul(o, sb[j]));
                    const uint32_t mo_b = qk::bf2_add(qk::bf2_mul(o, cb[j]), qk::bf2_mul(e, nb2[j]));
                    me = f2_make(bf16_lo(me_b), bf16_hi(me_b));
                    mo = f2_make(bf16_lo(mo_b), bf16_hi(mo_b));
                } else {
                    me = de[j];
                    mo = dd[j];
                    if constexpr (ROPE && V2) {  // bf16 products, their sums rounded below
                        me = f2_add(round_pair<T>(f2_mul(de[j], c2[j])), round_pair<T>(f2_mul(dd[j], s2[j])));
                        mo = f2_add(round_pair<T>(f2_mul(dd[j], c2[j])), round_pair<T>(f2_mul(de[j], n2[j])));
                    } else if constexpr (ROPE) {  // R^T: (c dy0 + s dy1, -s dy0 + c dy1)
                        me = f2_fma(dd[j], s2[j], f2_mul(de[j], c2[j]));
                        mo = f2_fma(de[j], n2[j], f2_mul(dd[j], c2[j]));
                    }
                    me = round_pair<T>(me);  // gradient of the rotated-in value, Q/K dtype
                    mo = round_pair<T>(mo);
                }
                if constexpr (SCALE) {   // through the query_scale cast
                    me = round_pair<T>(f2_mul(me, qs2));
                    mo = round_pair<T>(f2_mul(mo, qs2));
                }
                de[j] = me;
                dd[j] = mo;
                ss = f2_fma(xe[j], xe[j], ss);
                ss = f2_fma(xo[j], xo[j], ss);
                cd = f2_fma(me, xe[j], cd);
                cd = f2_fma(mo, xo[j], cd);
            }
            const float r = inv_rms_fast(group_sum<L>(f2_sum(ss)), inv_width, a.eps);
            const float cr = r * r * r * group_sum<L>(f2_sum(cd)) * inv_width;
            const f32x2 r2 = f2_make(r, r), ncr2 = f2_make(-cr, -cr);
#pragma unroll
            for (int j = 0; j < H; ++j) {
                de[j] = f2_fma(xe[j], ncr2, f2_mul(de[j], r2));
                dd[j] = f2_fma(xo[j], ncr2, f2_mul(dd[j], r2));
            }
            if (hv[b]) st_vec(dst + (uint32_t)(b * RW) * head_bytes + voff, qk::from_eo<T>(de, dd));
        }
    };

    bool alive = true;
    int64_t t = u0 / nb, cur_t = -1;
    int j = (int)(u0 - t * nb);
    int i = 0;
#pragma unroll 1
    for (; i < n; ++i) {
        alive = __all_sync(0xffffffffu, alive && pipe::mbar_wait(&bars[warp][i % R], (uint32_t)((i / R) & 1)));
        if (!alive) break;
        int st0, s_hi, count;
        bool isq;
        batch(j, st0, s_hi, count, isq);
        const unsigned char* sl = ring + (i % R) * slot_bytes + (uint32_t)slot * head_bytes + voff;
        uint4 xv[BATCH], gv[BATCH];
        bool hv[BATCH];
#pragma unroll
        for (int b = 0; b < BATCH; ++b) {
            hv[b] = vok && (!TAIL || (st0 + b < s_hi && (st0 + b) * RW + slot < count));
            const uint32_t o = (uint32_t)(b * RW) * head_bytes;
            xv[b] = hv[b] ? *reinterpret_cast<const uint4*>(sl + o) : make_uint4(0, 0, 0, 0);
            gv[b] = hv[b] ? *reinterpret_cast<const uint4*>(sl + half_slot + o) : make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
        if (lane == 0 && issued < n) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            issue(issued);
            ++issued;
        }
        if (t != cur_t) {
            set_angles(t);
            cur_t = t;
        }
        char* dst = isq ? static_cast<char*>(a.q_out) + t * a.q_out_stride * (int64_t)sizeof(T)
                        : static_cast<char*>(a.k_out) + t * a.k_out_stride * (int64_t)sizeof(T);
        dst += (uint32_t)slot * head_bytes + (uint32_t)(st0 * RW) * head_bytes;
        if (isq && scaled)
            compute(std::true_type{}, xv, gv, hv, dst);
        else
            compute(std::false_type{}, xv, gv, hv, dst);
        if (++j == nb) {
            j = 0;
            ++t;
        }
    }
    if (lane == 0)
        for (int k = i; k < issued; ++k)
            if (!pipe::mbar_wait(&bars[warp][k % R], (uint32_t)((k / R) & 1))) break;
}

constexpr int kThreads = 256;
constexpr int kBwdBatch = 4;
constexpr int kBwdRing = 2;

template <typename T, int L, int VPL>
cudaError_t launch_gate_head(const GateBwdArgs& a, cudaStream_t s) {
    constexpr int RW = 32 / L;
    const int64_t per_cta = (int64_t)(kThreads / 32) * RW;
    return launch_pdl(output_norm_gate_bwd_kernel<T, L, VPL>, (unsigned)((a.rows + per_cta - 1) / per_cta),
                      kThreads, 0, s, a);
}

template <typename T, int VPT>
cudaError_t launch_gate_group(const GateBwdArgs& a, int nvec, cudaStream_t s) {
    const int threads = ((nvec + VPT - 1) / VPT + 31) / 32 * 32;
    return launch_pdl(output_norm_gate_group_bwd_kernel<T, VPT>, (unsigned)a.rows, (unsigned)threads, 0, s, a);
}

template <typename T>
cudaError_t launch_gate_bwd_t(const GateBwdArgs& a, cudaStream_t s) {
    const int nv = a.width / Vec<T>::N;
    if (nv > 32) {
        if (nv <= 512) return launch_gate_group<T, 1>(a, nv, s);
        if (nv <= 1024) return launch_gate_group<T, 2>(a, nv, s);
        if (nv <= 2048) return launch_gate_group<T, 4>(a, nv, s);
        return launch_gate_group<T, 8>(a, nv, s);
    }
    if (nv >= 16) {
        const int lanes = (nv + 1) / 2;
        if (lanes <= 8) return launch_gate_head<T, 8, 2>(a, s);
        if (lanes <= 16) return launch_gate_head<T, 16, 2>(a, s);
        return launch_gate_head<T, 32, 1>(a, s);
    }
    if (nv <= 1) return launch_gate_head<T, 1, 1>(a, s);
    if (nv <= 2) return launch_gate_head<T, 2, 1>(a, s);
    if (nv <= 4) return launch_gate_head<T, 4, 1>(a, s);
    if (nv <= 8) return launch_gate_head<T, 8, 1>(a, s);
    return launch_gate_head<T, 16, 1>(a, s);
}

template <typename T, int L, bool ROPE, bool V2>
cudaError_t launch_qk_bwd_l(const QkBwdArgs& A, cudaStream_t s) {
    constexpr int RW = 32 / L;
    constexpr int BATCH = kBwdBatch;
    const QkArgs& a = A.f;
    const int nwarps = kThreads / 32;
    const int nst_q = (a.hq + RW - 1) / RW, nst_k = (a.hkv + RW - 1) / RW;
    const int64_t units = a.tokens * ((nst_q + BATCH - 1) / BATCH + (nst_k + BATCH - 1) / BATCH);
    const uint32_t head_bytes = (uint32_t)a.head_dim * (uint32_t)sizeof(T);
    const size_t half_slot = ((size_t)BATCH * RW * head_bytes + 127) & ~(size_t)127;
    const size_t smem = (size_t)nwarps * kBwdRing * 2 * half_slot;
    const bool exact = a.head_dim / Vec<T>::N == L && a.hq % RW == 0 && a.hkv % RW == 0 &&
                       nst_q % BATCH == 0 && nst_k % BATCH == 0;
    auto kern = exact ? qk_norm_rope_bwd_kernel<T, L, ROPE, V2, false, BATCH, kBwdRing>
                      : qk_norm_rope_bwd_kernel<T, L, ROPE, V2, true, BATCH, kBwdRing>;
    // the opt-in is needed whenever static + dynamic shared memory passes 48 KB
    // (the mbarriers are static), so it is always set
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int64_t grid = (int64_t)blocks_per_sm((const void*)kern, kThreads, smem) * sm_count();
    const int64_t need = (units + nwarps - 1) / nwarps;
    if (grid > need) grid = need;
    if (grid < 1) grid = 1;
    return launch_pdl(kern, (unsigned)grid, kThreads, smem, s, A);
}

template <typename T, int L>
cudaError_t launch_qk_bwd_r(int use_rope, int upcast, const QkBwdArgs& a, cudaStream_t s) {
    if (!use_rope) return launch_qk_bwd_l<T, L, false, false>(a, s);
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        if (!upcast) return launch_qk_bwd_l<T, L, true, true>(a, s);
    }
    return launch_qk_bwd_l<T, L, true, false>(a, s);
}

template <typename T>
cudaError_t launch_qk_bwd_t(int use_rope, int upcast, const QkBwdArgs& a, cudaStream_t s) {
    const int nv = a.f.head_dim / Vec<T>::N;
    if (nv > 16) return launch_qk_bwd_r<T, 32>(use_rope, upcast, a, s);
    if (nv <= 1) return launch_qk_bwd_r<T, 1>(use_rope, upcast, a, s);
    if (nv <= 2) return launch_qk_bwd_r<T, 2>(use_rope, upcast, a, s);
    if (nv <= 4) return launch_qk_bwd_r<T, 4>(use_rope, upcast, a, s);
    if (nv <= 8) return launch_qk_bwd_r<T, 8>(use_rope, upcast, a, s);
    return launch_qk_bwd_r<T, 16>(use_rope, upcast, a, s);
}

}  // namespace

cudaError_t launch_gate_bwd(int dtype, const GateBwdArgs& a, cudaStream_t s) {
    return dtype == 0 ? launch_gate_bwd_t<__nv_bfloat16>(a, s) : launch_gate_bwd_t<float>(a, s);
}

cudaError_t launch_qk_bwd(int dtype, int use_rope, int upcast_rope, const QkBwdArgs& a, cudaStream_t s) {
    // FP32 tensors rotate in FP32 in both modes.
    return dtype == 0 ? launch_qk_bwd_t<__nv_bfloat16>(use_rope, upcast_rope, a, s)
                      : launch_qk_bwd_t<float>(use_rope, 1, a, s);
}

cudaError_t read_qk_bwd_device_error(unsigned int* out, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_device_error, sizeof(unsigned int));
    if (e == cudaSuccess && clear) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned int));
    }
    return e;
}

}  // namespace muse
