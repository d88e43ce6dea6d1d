// Row-wide normalisation kernels: cores 1, 2, 5 and core 4 with one norm per
// token.  One CTA normalises one row at a time, NT threads x VPT 16-byte slots
// covering the row, and owns a chunk of rows_per_cta consecutive rows (one
// to four consecutive rows: a one-shot grid of small CTAs, which streams best
// on B200 - measured against persistent grids; core 5's per-channel cos/sin
// of the blend angle are computed once per thread and reused over its chunk).  Within a chunk a ring of S
// row buffers in registers keeps the next rows' loads in flight while the
// current row is reduced and written.
#include "common.cuh"
#include "kernels.h"

namespace muse {
namespace {

constexpr int kMaxThreads = 512;  // threads per CTA (one row)
constexpr int kResidualChunk = 4;  // rows per CTA for core 5
constexpr int kRowChunk = 2;       // rows per CTA for cores 1, 2 and 4

__host__ __device__ constexpr bool is_residual(RowOp op) { return op == RowOp::kResidual || op == RowOp::kResidualIS; }
__host__ __device__ constexpr bool scales_first(RowOp op) { return op == RowOp::kInputScale || op == RowOp::kResidualIS; }

template <typename T, RowOp OP, int VPT>
struct RowFrag {
    static constexpr int V = Vec<T>::N;
    static constexpr int SV = V / 4;  // 16-byte FP32 stream vectors per slot
    uint4 x[VPT];
    uint4 g[OP == RowOp::kNormGate ? VPT : 1];
    uint4 h[is_residual(OP) ? VPT * SV : 1];
};

template <typename T, RowOp OP, int VPT, bool HAS_GAIN, int STAGES>
__device__ __forceinline__ void row_norm_body(const RowArgs& a) {
    constexpr int V = Vec<T>::N;
    constexpr int SV = V / 4;
    using Frag = RowFrag<T, OP, VPT>;
    __shared__ float red[2][32];

    const int tid = threadIdx.x;
    const int nt = blockDim.x;
    const int nvec = a.width / V;
    const float widthf = (float)a.width;

    bool valid[VPT];
#pragma unroll
    for (int i = 0; i < VPT; ++i) valid[i] = tid + i * nt < nvec;

    // Per-slot constants, fixed for the CTA's lifetime: effective gain
    // (16-byte loads) and the blend's cos/sin.
    float w[HAS_GAIN ? VPT : 1][V];
    float cth[is_residual(OP) ? VPT : 1][V];
    float sth[is_residual(OP) ? VPT : 1][V];
    auto load_constants = [&]() {
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = valid[i] ? tid + i * nt : 0;
            if constexpr (HAS_GAIN) {
#pragma unroll
                for (int k = 0; k < V / 4; ++k) {
                    const float4 g4 = __ldg(reinterpret_cast<const float4*>(a.gain) + v * (V / 4) + k);
                    w[i][4 * k + 0] = g4.x + a.gain_offset;
                    w[i][4 * k + 1] = g4.y + a.gain_offset;
                    w[i][4 * k + 2] = g4.z + a.gain_offset;
                    w[i][4 * k + 3] = g4.w + a.gain_offset;
                }
            }
            if constexpr (is_residual(OP)) {
#pragma unroll
                for (int k = 0; k < V / 4; ++k) {
                    const float4 t4 = __ldg(reinterpret_cast<const float4*>(a.theta) + v * (V / 4) + k);
                    const float th[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) sincosf(th[e], &sth[i][4 * k + e], &cth[i][4 * k + e]);
                }
            }
        }
    };

    auto load = [&](int64_t row, Frag& f) {
        const char* xr = static_cast<const char*>(a.x) + row * a.x_stride * (int64_t)sizeof(T);
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = tid + i * nt;
            f.x[i] = valid[i] ? ld_stream(xr + (int64_t)v * 16) : make_uint4(0, 0, 0, 0);
            if constexpr (OP == RowOp::kNormGate) {
                const char* gr = static_cast<const char*>(a.gate) + row * a.gate_stride * (int64_t)sizeof(T);
                f.g[i] = valid[i] ? ld_stream(gr + (int64_t)v * 16) : make_uint4(0, 0, 0, 0);
            }
            if constexpr (is_residual(OP)) {
                const char* hr = reinterpret_cast<const char*>(a.stream_in + row * a.s_in_stride);
#pragma unroll
                for (int k = 0; k < SV; ++k)
                    f.h[i * SV + k] = valid[i] ? ld_stream(hr + ((int64_t)v * SV + k) * 16)
                                               : make_uint4(0, 0, 0, 0);
            }
        }
    };

    auto process = [&](int64_t row, const Frag& f, int& bank) {
        float xf[VPT][V];
        float ss = 0.0f;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            unpack<T>(f.x[i], xf[i]);
            if constexpr (scales_first(OP) && HAS_GAIN) {
#pragma unroll
                for (int e = 0; e < V; ++e) xf[i][e] = xf[i][e] * w[i][e];
            }
            ss += sum_sq<V>(xf[i]);
        }
        const float r = inv_rms(block_sum(ss, red, bank), widthf, a.eps);

        if constexpr (OP == RowOp::kRms || OP == RowOp::kInputScale || OP == RowOp::kNormGate) {
            char* yr = static_cast<char*>(a.y) + row * a.y_stride * (int64_t)sizeof(T);
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                float o[V];
                float gf[V];
                if constexpr (OP == RowOp::kNormGate) unpack<T>(f.g[i], gf);
#pragma unroll
                for (int e = 0; e < V; ++e) {
                    float t = xf[i][e] * r;
                    if constexpr (OP == RowOp::kRms && HAS_GAIN) t = t * w[i][e];
                    if constexpr (OP == RowOp::kNormGate) t = times_sigmoid<T>(t, gf[e]);
                    o[e] = t;
                }
                if (valid[i]) st_vec(yr + (int64_t)(tid + i * nt) * 16, pack<T>(o));
            }
        } else {
            char* hr = reinterpret_cast<char*>(a.stream_out + row * a.s_out_stride);
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                float hin[V];
#pragma unroll
                for (int k = 0; k < SV; ++k) unpack<float>(f.h[i * SV + k], hin + 4 * k);
                float o[V];
#pragma unroll
                for (int e = 0; e < V; ++e) {
                    float t = xf[i][e] * r;  // z r when the gain came first
                    if constexpr (OP == RowOp::kResidual && HAS_GAIN) t = t * w[i][e];
                    const float nb = round_to<T>(t);  // cast back to the branch dtype
                    o[e] = cth[i][e] * hin[e] + sth[i][e] * nb;
                }
                if (valid[i]) {
#pragma unroll
                    for (int k = 0; k < SV; ++k)
                        st_vec(hr + ((int64_t)(tid + i * nt) * SV + k) * 16, pack<float>(o + 4 * k));
                }
            }
        }
    };

    // This CTA's rows [r0, r1); a ring of STAGES row buffers.
    const int64_t r0 = (int64_t)blockIdx.x * a.rows_per_cta;
    const int64_t r1 = min(r0 + (int64_t)a.rows_per_cta, a.rows);
    Frag f[STAGES];
#pragma unroll
    for (int s = 0; s < STAGES; ++s)
        if (r0 + s < r1) load(r0 + s, f[s]);
    load_constants();  // overlaps the first loads
    int bank = 0;
    for (int64_t base = r0; base < r1; base += STAGES) {
#pragma unroll
        for (int s = 0; s < STAGES; ++s) {
            const int64_t r = base + s;
            if (r < r1) {  // uniform across the CTA
                process(r, f[s], bank);
                if (r + STAGES < r1) load(r + STAGES, f[s]);
            }
        }
    }
}

// One entry symbol per core, so launch lists and profiles name the core.
template <typename T, int VPT, bool G, int S>
__global__ void __launch_bounds__(kMaxThreads) rms_norm_kernel(const __grid_constant__ RowArgs a) {
    row_norm_body<T, RowOp::kRms, VPT, G, S>(a);
}
template <typename T, int VPT, bool G, int S>
__global__ void __launch_bounds__(kMaxThreads) input_scale_norm_kernel(const __grid_constant__ RowArgs a) {
    row_norm_body<T, RowOp::kInputScale, VPT, G, S>(a);
}
template <typename T, int VPT, bool G, int S>
__global__ void __launch_bounds__(kMaxThreads) output_norm_gate_row_kernel(const __grid_constant__ RowArgs a) {
    row_norm_body<T, RowOp::kNormGate, VPT, G, S>(a);
}
template <typename T, int VPT, bool G, int S>
__global__ void __launch_bounds__(kMaxThreads) norm_residual_kernel(const __grid_constant__ RowArgs a) {
    row_norm_body<T, RowOp::kResidual, VPT, G, S>(a);
}
template <typename T, int VPT, bool G, int S>
__global__ void __launch_bounds__(kMaxThreads) norm_residual_input_scale_kernel(const __grid_constant__ RowArgs a) {
    row_norm_body<T, RowOp::kResidualIS, VPT, G, S>(a);
}

// Row buffers in the ring: one.  Measured on B200 (prefill rows, H = 4096):
// deeper rings cost occupancy and lose to more resident CTAs.
template <RowOp OP>
constexpr int stages() { return 1; }

template <typename T, RowOp OP, int VPT, bool G>
constexpr auto row_kernel() {
    constexpr int S = stages<OP>();
    if constexpr (OP == RowOp::kRms) return rms_norm_kernel<T, VPT, G, S>;
    else if constexpr (OP == RowOp::kInputScale) return input_scale_norm_kernel<T, VPT, G, S>;
    else if constexpr (OP == RowOp::kNormGate) return output_norm_gate_row_kernel<T, VPT, G, S>;
    else if constexpr (OP == RowOp::kResidual) return norm_residual_kernel<T, VPT, G, S>;
    else return norm_residual_input_scale_kernel<T, VPT, G, S>;
}

template <typename T, RowOp OP, int VPT>
cudaError_t launch_row_vpt(const RowArgs& a0, int nvec, cudaStream_t s) {
    RowArgs a = a0;
    const int nt = ((nvec + VPT - 1) / VPT + 31) / 32 * 32;
    a.rows_per_cta = is_residual(OP) ? kResidualChunk : kRowChunk;
    auto kern = a.gain ? row_kernel<T, OP, VPT, true>() : row_kernel<T, OP, VPT, false>();
    const int64_t grid = (a.rows + a.rows_per_cta - 1) / a.rows_per_cta;
    kern<<<(unsigned)grid, nt, 0, s>>>(a);
    return cudaGetLastError();
}

// Slots per thread: the fewest that fit a row into kThreadsRow threads (small
// CTAs, many resident) - or kMaxThreads for core 5, whose per-thread cos/sin
// registers favour fewer slots.
constexpr int kThreadsRow = 128;

template <typename T, RowOp OP>
cudaError_t launch_row_t(const RowArgs& a, cudaStream_t s) {
    const int nvec = a.width / Vec<T>::N;
    const int cap = is_residual(OP) ? kMaxThreads : kThreadsRow;
    if (nvec <= cap) return launch_row_vpt<T, OP, 1>(a, nvec, s);
    if (nvec <= 2 * cap) return launch_row_vpt<T, OP, 2>(a, nvec, s);
    if (nvec <= 4 * cap) return launch_row_vpt<T, OP, 4>(a, nvec, s);
    return launch_row_vpt<T, OP, 8>(a, nvec, s);
}

template <typename T>
cudaError_t launch_row_dt(RowOp op, const RowArgs& a, cudaStream_t s) {
    switch (op) {
        case RowOp::kRms: return launch_row_t<T, RowOp::kRms>(a, s);
        case RowOp::kInputScale: return launch_row_t<T, RowOp::kInputScale>(a, s);
        case RowOp::kNormGate: return launch_row_t<T, RowOp::kNormGate>(a, s);
        case RowOp::kResidual: return launch_row_t<T, RowOp::kResidual>(a, s);
        case RowOp::kResidualIS: return launch_row_t<T, RowOp::kResidualIS>(a, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_row(int dtype, RowOp op, const RowArgs& a, cudaStream_t s) {
    return dtype == 0 ? launch_row_dt<__nv_bfloat16>(op, a, s) : launch_row_dt<float>(op, a, s);
}

}  // namespace muse
