// _residual_core / MuseSparkResidual.forward: the FP32 residual stream blended
// with the branch as it arrives (no branch norm), per channel
//   stream_out = c * stream_in + s * f32(branch),
// with (c, s) = (cos theta, sin theta) - the blend core 5 uses - or, from the
// learned gate, c^2 = max(sigmoid(gate / temperature), eps), s^2 = 1 - c^2
// (the same blend with theta = atan2(s, c)).
//
// Purely elementwise, so no shared-memory staging: each thread owns one
// 16-byte vector of branch columns (and the matching 32 or 16 bytes of the
// stream) for the whole launch, computes its columns' coefficients once into
// registers, and walks the tiles of U consecutive rows dealt to its CTA
// (round-robin over the grid), issuing the loads of a tile before any
// arithmetic.  2-D grid: y covers the
// columns in blocks of the CTA width, x the rows (resident CTAs x SMs in all).
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace muse {
namespace {

constexpr int kBlendRows = 8;  // rows in flight per thread (4: 5% slower; a 4-CTA register cap: slower)

// The gate form's two coefficients of one channel: x = gate / temperature,
// t = |x|.  The larger coefficient is sqrt(sigmoid(t)) = 1 / sqrt(1 + e^-t),
// the smaller one sqrt(sigmoid(-t)) = e^(-t/2) / sqrt(1 + e^-t) (no
// subtraction from 1, no underflow of sigmoid(-t)); then the bound
// c^2 >= eps, i.e. c >= sqrt(eps) and s <= sqrt(1 - eps).
template <typename F>
__device__ __forceinline__ void gate_coefficients(const ResidualArgs& a, float g, F& c, F& s) {
    const F x = (F)g / (F)a.temperature;
    const F t = fabs(x);
    const F big = (F)1 / sqrt((F)1 + exp(-t));
    const F small = exp((F)-0.5 * t) * big;
    c = fmax(x >= (F)0 ? big : small, sqrt((F)a.eps));
    s = fmin(x >= (F)0 ? small : big, sqrt((F)1 - (F)a.eps));
}

// The blend's two coefficients of one channel: from the gate (FP32: the
// small coefficient carries the FP32 rounding of x, up to |x| 2^-25
// relative, but it weighs e^(-|x|/2) against a coefficient near 1, so its
// share of the result's error stays far below 2e-6 of the terms), or cos and
// sin of the FP32 angle.
template <bool GATE>
__device__ __forceinline__ void blend_coefficients(const ResidualArgs& a, float p, float& c, float& s) {
    if constexpr (GATE) {
        gate_coefficients<float>(a, p, c, s);
    } else {
        sincosf(p, &s, &c);
    }
}

template <typename T, bool GATE>
__global__ void __launch_bounds__(256) residual_blend_kernel(const __grid_constant__ ResidualArgs a) {
    pdl_begin();
    constexpr int V = Vec<T>::N;   // branch elements per 16-byte vector
    constexpr int SV = V / 4;      // 16-byte FP32 stream pieces per vector
    constexpr int P = V / 2;       // packed FP32 pairs per vector
    constexpr int U = kBlendRows;
    const int64_t cv = (int64_t)blockIdx.y * blockDim.x + threadIdx.x;  // this thread's vector column
    if (cv * V >= a.width) return;
    const int64_t col = cv * V;

    f32x2 c2[P], s2[P];
    {
        const float* src = GATE ? a.gate : a.theta;
#pragma unroll
        for (int q = 0; q < SV; ++q) {
            const float4 p4 = __ldg(reinterpret_cast<const float4*>(src + col) + q);
            float c0, s0, c1, s1, c2_, s2_, c3, s3;
            blend_coefficients<GATE>(a, p4.x, c0, s0);
            blend_coefficients<GATE>(a, p4.y, c1, s1);
            blend_coefficients<GATE>(a, p4.z, c2_, s2_);
            blend_coefficients<GATE>(a, p4.w, c3, s3);
            c2[2 * q] = f2_make(c0, c1);
            c2[2 * q + 1] = f2_make(c2_, c3);
            s2[2 * q] = f2_make(s0, s1);
            s2[2 * q + 1] = f2_make(s2_, s3);
        }
    }

    const char* b_base = static_cast<const char*>(a.branch) + col * (int64_t)sizeof(T);
    const float* h_base = a.stream_in + col;
    float* o_base = a.stream_out + col;
    // tiles of U consecutive rows, dealt round-robin over the grid: at any time
    // the grid streams one compact window of the tensors
    for (int64_t r0 = (int64_t)blockIdx.x * U; r0 < a.rows; r0 += (int64_t)gridDim.x * U) {
        uint4 bv[U], hv[U][SV];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t row = r0 + u;
            const bool ok = row < a.rows;
            bv[u] = ok ? ld_stream(b_base + row * a.width * (int64_t)sizeof(T)) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int q = 0; q < SV; ++q)
                hv[u][q] = ok ? ld_stream(h_base + row * a.width + 4 * q) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t row = r0 + u;
            f32x2 b[P], h[P], o[P];
            to_pairs<T>(bv[u], b);
#pragma unroll
            for (int q = 0; q < SV; ++q) to_pairs<float>(hv[u][q], h + 2 * q);
#pragma unroll
            for (int q = 0; q < P; ++q) o[q] = f2_fma(c2[q], h[q], f2_mul(s2[q], b[q]));
            if (row < a.rows) {
#pragma unroll
                for (int q = 0; q < SV; ++q) st_vec(o_base + row * a.width + 4 * q, from_pairs<float>(o + 2 * q));
            }
        }
    }
}

// The blend angle of each channel from the gate: theta = atan2(s, c), in
// double and rounded once - the angle alone is the output here, and the
// smaller coefficient (so theta near 0 or pi/2) is exponentially sensitive to
// x: an FP32 rounding of x = 150 alone moves e^(-x/2) by 4e-6 relative.
__global__ void __launch_bounds__(256) residual_gate_angles_kernel(const __grid_constant__ ResidualArgs a,
                                                                   float* theta) {
    pdl_begin();
    const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= a.width) return;
    double c, s;
    gate_coefficients<double>(a, __ldg(a.gate + j), c, s);
    theta[j] = (float)atan2(s, c);
}

// Backward: per row, dstream = c dy (FP32), dbranch = cast(s dy); per column
// the angle gradient sum dy (c b - s h), or for the gate the sum
// dy (s h - c b) times c s / (2 temperature) (zero where eps bounds c),
// accumulated over the thread's rows in registers and written as one partial
// row per CTA row-block into the caller's workspace (a fixed-order reduction
// follows).
constexpr int kBlendBwdRows = 8;  // rows in flight per thread (4: 14% slower, 2: 16% slower)

template <typename T, bool GATE>
__global__ void __launch_bounds__(256) residual_blend_bwd_kernel(const __grid_constant__ ResidualArgs a) {
    pdl_begin();
    constexpr int V = Vec<T>::N;
    constexpr int SV = V / 4;
    constexpr int P = V / 2;
    constexpr int U = kBlendBwdRows;
    const int64_t cv = (int64_t)blockIdx.y * blockDim.x + threadIdx.x;
    if (cv * V >= a.width) return;
    const int64_t col = cv * V;

    f32x2 c2[P], s2[P], ns2[P], k2[P];
    {
        const float* src = GATE ? a.gate : a.theta;
        float cf[V], sf[V], kf[V];
#pragma unroll
        for (int q = 0; q < SV; ++q) {
            const float4 p4 = __ldg(reinterpret_cast<const float4*>(src + col) + q);
            const float pv[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                blend_coefficients<GATE>(a, pv[e], cf[4 * q + e], sf[4 * q + e]);
                kf[4 * q + e] = 1.0f;
                if constexpr (GATE) {
                    // dc/dgate = c s^2 / (2 temperature), ds/dgate = -s c^2 / (2 temperature):
                    // the gate gradient is k (s h - c b) dy with k = c s / (2 temperature);
                    // zero where the bound holds c (sigmoid(gate / temperature) < eps)
                    const float x = pv[e] / a.temperature;
                    const float cu = x >= 0.0f ? 1.0f / sqrtf(1.0f + expf(-x)) : expf(0.5f * x) / sqrtf(1.0f + expf(x));
                    kf[4 * q + e] = cu >= sqrtf(a.eps) ? cf[4 * q + e] * sf[4 * q + e] / (2.0f * a.temperature) : 0.0f;
                }
            }
        }
#pragma unroll
        for (int q = 0; q < P; ++q) {
            c2[q] = f2_make(cf[2 * q], cf[2 * q + 1]);
            s2[q] = f2_make(sf[2 * q], sf[2 * q + 1]);
            ns2[q] = f2_make(-sf[2 * q], -sf[2 * q + 1]);
            k2[q] = f2_make(kf[2 * q], kf[2 * q + 1]);
        }
    }

    f32x2 acc[P];
#pragma unroll
    for (int q = 0; q < P; ++q) acc[q] = f2_make(0.0f, 0.0f);
    const char* b_base = static_cast<const char*>(a.branch) + col * (int64_t)sizeof(T);
    const float* h_base = a.stream_in + col;
    const float* g_base = a.dy + col;
    float* dh_base = a.stream_out + col;  // dstream
    char* db_base = static_cast<char*>(a.dbranch) + col * (int64_t)sizeof(T);
    for (int64_t r0 = (int64_t)blockIdx.x * U; r0 < a.rows; r0 += (int64_t)gridDim.x * U) {
        uint4 bv[U], hv[U][SV], gv[U][SV];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t row = r0 + u;
            const bool ok = row < a.rows;
            bv[u] = ok ? ld_stream(b_base + row * a.width * (int64_t)sizeof(T)) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int q = 0; q < SV; ++q) {
                hv[u][q] = ok ? ld_stream(h_base + row * a.width + 4 * q) : make_uint4(0, 0, 0, 0);
                gv[u][q] = ok ? ld_stream(g_base + row * a.width + 4 * q) : make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t row = r0 + u;
            f32x2 b[P], h[P], g[P], dh[P], db[P];
            to_pairs<T>(bv[u], b);
#pragma unroll
            for (int q = 0; q < SV; ++q) {
                to_pairs<float>(hv[u][q], h + 2 * q);
                to_pairs<float>(gv[u][q], g + 2 * q);
            }
#pragma unroll
            for (int q = 0; q < P; ++q) {
                dh[q] = f2_mul(c2[q], g[q]);
                db[q] = f2_mul(s2[q], g[q]);
                // angle: dy (c b - s h); gate: dy (s h - c b), scaled by k at the end
                const f32x2 t = GATE ? f2_fma(s2[q], h[q], f2_mul(f2_make(-1.0f, -1.0f), f2_mul(c2[q], b[q])))
                                     : f2_fma(c2[q], b[q], f2_mul(ns2[q], h[q]));
                acc[q] = f2_fma(g[q], t, acc[q]);  // rows with row >= rows load zeros: no contribution
            }
            if (row < a.rows) {
#pragma unroll
                for (int q = 0; q < SV; ++q) st_vec(dh_base + row * a.width + 4 * q, from_pairs<float>(dh + 2 * q));
                st_vec(db_base + row * a.width * (int64_t)sizeof(T), from_pairs<T>(db));
            }
        }
    }
    if (a.part) {
        float* out = a.part + (int64_t)blockIdx.x * a.width + col;
#pragma unroll
        for (int q = 0; q < P; ++q) acc[q] = f2_mul(acc[q], k2[q]);
#pragma unroll
        for (int q = 0; q < SV; ++q) st_vec(out + 4 * q, from_pairs<float>(acc + 2 * q));
    }
}

template <typename T, bool GATE>
cudaError_t launch_blend(const ResidualArgs& a, cudaStream_t s) {
    constexpr int V = Vec<T>::N;
    const int64_t nvec = a.width / V;
    const int threads = nvec >= 256 ? 256 : (int)((nvec + 31) / 32 * 32);
    const int64_t gy = (nvec + threads - 1) / threads;
    auto kern = residual_blend_kernel<T, GATE>;
    const int64_t ctas = (int64_t)blocks_per_sm((const void*)kern, threads) * sm_count();
    int64_t gx = (ctas + gy - 1) / gy;
    if (gx > (a.rows + kBlendRows - 1) / kBlendRows) gx = (a.rows + kBlendRows - 1) / kBlendRows;
    if (gx < 1) gx = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)gx, (unsigned)gy);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

// Grid of the backward: resident CTAs as column blocks x row blocks (each row
// block writes one partial row).  With plan_only the kernel is not launched.
template <typename T, bool GATE>
cudaError_t launch_blend_bwd(ResidualArgs a, float* dparam, cudaStream_t s, int64_t* plan_gx) {
    constexpr int V = Vec<T>::N;
    const int64_t nvec = a.width / V;
    const int threads = nvec >= 256 ? 256 : (int)((nvec + 31) / 32 * 32);
    const int64_t gy = (nvec + threads - 1) / threads;
    auto kern = residual_blend_bwd_kernel<T, GATE>;
    const int64_t ctas = (int64_t)blocks_per_sm((const void*)kern, threads) * sm_count();
    int64_t gx = (ctas + gy - 1) / gy;
    const int64_t tiles = (a.rows + kBlendBwdRows - 1) / kBlendBwdRows;
    if (gx > tiles) gx = tiles;
    if (gx < 1) gx = 1;
    if (plan_gx) {
        *plan_gx = gx;
        return cudaSuccess;
    }
    if (!dparam) a.part = nullptr;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)gx, (unsigned)gy);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a);
    if (e != cudaSuccess || !dparam) return e;
    return launch_param_grad_reduce(a.part, (int)gx, (int)a.width, dparam, s);
}

}  // namespace

cudaError_t launch_residual_blend_bwd(int dtype, bool gate, const ResidualArgs& a, float* dparam,
                                      cudaStream_t s, int64_t* plan_gx) {
    if (dtype == 0)
        return gate ? launch_blend_bwd<__nv_bfloat16, true>(a, dparam, s, plan_gx)
                    : launch_blend_bwd<__nv_bfloat16, false>(a, dparam, s, plan_gx);
    return gate ? launch_blend_bwd<float, true>(a, dparam, s, plan_gx)
                : launch_blend_bwd<float, false>(a, dparam, s, plan_gx);
}

cudaError_t launch_residual_blend(int dtype, bool gate, const ResidualArgs& a, cudaStream_t s) {
    if (dtype == 0)
        return gate ? launch_blend<__nv_bfloat16, true>(a, s) : launch_blend<__nv_bfloat16, false>(a, s);
    return gate ? launch_blend<float, true>(a, s) : launch_blend<float, false>(a, s);
}

cudaError_t launch_residual_gate_angles(const ResidualArgs& a, float* theta, cudaStream_t s) {
    const unsigned grid = (unsigned)((a.width + 255) / 256);
    return launch_pdl(residual_gate_angles_kernel, grid, 256u, 0, s, a, theta);
}

}  // namespace muse
