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
constexpr int kResidualChunk = 8;  // rows per CTA for core 5
constexpr int kRowChunk = 4;       // rows per CTA for cores 1, 2 and 4

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

// Per-thread constant pieces (float4) per slot: effective gain, cos, sin.
template <typename T, RowOp OP, bool HAS_GAIN>
__host__ __device__ constexpr int const_pieces_per_slot() {
    return (HAS_GAIN ? Vec<T>::N / 4 : 0) + (is_residual(OP) ? 2 * (Vec<T>::N / 4) : 0);
}

// CSM: the constants live in shared memory (each thread reads back only what
// it wrote, so no barrier) instead of registers - fewer registers, more
// resident CTAs, more rows in flight.
template <typename T, RowOp OP, int VPT, bool HAS_GAIN, int STAGES, bool CSM>
__device__ __forceinline__ void row_norm_body(const RowArgs& a) {
    constexpr int V = Vec<T>::N;
    constexpr int SV = V / 4;
    constexpr int CP = const_pieces_per_slot<T, OP, HAS_GAIN>();
    constexpr int GOFF = 0, COFF = HAS_GAIN ? SV : 0, SOFF = COFF + SV;
    using Frag = RowFrag<T, OP, VPT>;
    __shared__ float red[2][32];
    extern __shared__ float4 csm[];  // [VPT * CP][nt] when CSM

    const int tid = threadIdx.x;
    const int nt = blockDim.x;
    const int nvec = a.width / V;
    const float inv_width = 1.0f / (float)a.width;

    bool valid[VPT];
#pragma unroll
    for (int i = 0; i < VPT; ++i) valid[i] = tid + i * nt < nvec;

    // Per-slot constants, fixed for the CTA's lifetime: effective gain
    // (16-byte loads) and the blend's cos/sin (computed, or read from a
    // [cos | sin] table when the caller provides one).
    constexpr int RV = CSM ? 1 : V;
    float w[HAS_GAIN ? VPT : 1][RV];
    float cth[is_residual(OP) ? VPT : 1][RV];
    float sth[is_residual(OP) ? VPT : 1][RV];
    auto put = [&](int i, int q, float4 v, float (&dst)[is_residual(OP) ? VPT : 1][RV], int k) {
        if constexpr (CSM) {
            csm[(i * CP + q) * nt + tid] = v;
        } else {
            dst[i][4 * k + 0] = v.x; dst[i][4 * k + 1] = v.y; dst[i][4 * k + 2] = v.z; dst[i][4 * k + 3] = v.w;
        }
    };
    auto load_constants = [&]() {
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = valid[i] ? tid + i * nt : 0;
#pragma unroll
            for (int k = 0; k < SV; ++k) {
                if constexpr (HAS_GAIN) {
                    float4 g4 = __ldg(reinterpret_cast<const float4*>(a.gain) + v * SV + k);
                    g4.x += a.gain_offset; g4.y += a.gain_offset; g4.z += a.gain_offset; g4.w += a.gain_offset;
                    if constexpr (CSM) {
                        csm[(i * CP + GOFF + k) * nt + tid] = g4;
                    } else {
                        w[i][4 * k + 0] = g4.x; w[i][4 * k + 1] = g4.y; w[i][4 * k + 2] = g4.z; w[i][4 * k + 3] = g4.w;
                    }
                }
                if constexpr (is_residual(OP)) {
                    float4 c4, s4;
                    if (a.cos_sin) {  // precomputed [cos | sin] table
                        c4 = __ldg(reinterpret_cast<const float4*>(a.cos_sin) + v * SV + k);
                        s4 = __ldg(reinterpret_cast<const float4*>(a.cos_sin + a.width) + v * SV + k);
                    } else {
                        const float4 t4 = __ldg(reinterpret_cast<const float4*>(a.theta) + v * SV + k);
                        sincosf(t4.x, &s4.x, &c4.x);
                        sincosf(t4.y, &s4.y, &c4.y);
                        sincosf(t4.z, &s4.z, &c4.z);
                        sincosf(t4.w, &s4.w, &c4.w);
                    }
                    put(i, COFF + k, c4, cth, k);
                    put(i, SOFF + k, s4, sth, k);
                }
            }
        }
    };
    // 4 constants of slot i, group k (elements 4k .. 4k+3)
    auto piece = [&](int i, int q, const float (&src)[is_residual(OP) ? VPT : 1][RV], int k) -> float4 {
        if constexpr (CSM) return csm[(i * CP + q) * nt + tid];
        else return make_float4(src[i][4 * k], src[i][4 * k + 1], src[i][4 * k + 2], src[i][4 * k + 3]);
    };
    auto wpiece = [&](int i, int k) -> float4 {
        if constexpr (CSM) return csm[(i * CP + GOFF + k) * nt + tid];
        else return make_float4(w[i][4 * k], w[i][4 * k + 1], w[i][4 * k + 2], w[i][4 * k + 3]);
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
                for (int k = 0; k < SV; ++k) {
                    const float4 w4 = wpiece(i, k);
                    xf[i][4 * k] *= w4.x; xf[i][4 * k + 1] *= w4.y; xf[i][4 * k + 2] *= w4.z; xf[i][4 * k + 3] *= w4.w;
                }
            }
            ss += sum_sq<V>(xf[i]);
        }
        const float r = inv_rms_fast(block_sum(ss, red, bank), inv_width, a.eps);

        if constexpr (OP == RowOp::kRms || OP == RowOp::kInputScale || OP == RowOp::kNormGate) {
            char* yr = static_cast<char*>(a.y) + row * a.y_stride * (int64_t)sizeof(T);
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                float o[V];
                float gf[V];
                if constexpr (OP == RowOp::kNormGate) unpack<T>(f.g[i], gf);
#pragma unroll
                for (int k = 0; k < SV; ++k) {
                    float4 w4 = make_float4(1.f, 1.f, 1.f, 1.f);
                    if constexpr (OP == RowOp::kRms && HAS_GAIN) w4 = wpiece(i, k);
                    const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int e = 4 * k + j;
                        float t = xf[i][e] * r;
                        if constexpr (OP == RowOp::kRms && HAS_GAIN) t = t * wv[j];
                        if constexpr (OP == RowOp::kNormGate) t = times_sigmoid<T>(t, gf[e]);
                        o[e] = t;
                    }
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
                for (int k = 0; k < SV; ++k) {
                    float4 w4 = make_float4(1.f, 1.f, 1.f, 1.f);
                    if constexpr (OP == RowOp::kResidual && HAS_GAIN) w4 = wpiece(i, k);
                    const float4 c4 = piece(i, COFF + k, cth, k), s4 = piece(i, SOFF + k, sth, k);
                    const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
                    const float cv[4] = {c4.x, c4.y, c4.z, c4.w}, sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int e = 4 * k + j;
                        float t = xf[i][e] * r;  // z r when the gain came first
                        if constexpr (OP == RowOp::kResidual && HAS_GAIN) t = t * wv[j];
                        const float nb = round_to<T>(t);  // cast back to the branch dtype
                        o[e] = cv[j] * hin[e] + sv[j] * nb;
                    }
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
template <typename T, int VPT, bool G, int S, bool CSM>
__global__ void __launch_bounds__(kMaxThreads) rms_norm_regs_kernel(const __grid_constant__ RowArgs a) {
    pdl_begin();
    row_norm_body<T, RowOp::kRms, VPT, G, S, CSM>(a);
}
template <typename T, int VPT, bool G, int S, bool CSM>
__global__ void __launch_bounds__(kMaxThreads) input_scale_norm_regs_kernel(const __grid_constant__ RowArgs a) {
    pdl_begin();
    row_norm_body<T, RowOp::kInputScale, VPT, G, S, CSM>(a);
}
template <typename T, int VPT, bool G, int S, bool CSM>
__global__ void __launch_bounds__(kMaxThreads) output_norm_gate_row_regs_kernel(const __grid_constant__ RowArgs a) {
    pdl_begin();
    row_norm_body<T, RowOp::kNormGate, VPT, G, S, CSM>(a);
}
template <typename T, int VPT, bool G, int S, bool CSM>
__global__ void __launch_bounds__(kMaxThreads) norm_residual_regs_kernel(const __grid_constant__ RowArgs a) {
    pdl_begin();
    row_norm_body<T, RowOp::kResidual, VPT, G, S, CSM>(a);
}
template <typename T, int VPT, bool G, int S, bool CSM>
__global__ void __launch_bounds__(kMaxThreads) norm_residual_input_scale_regs_kernel(const __grid_constant__ RowArgs a) {
    pdl_begin();
    row_norm_body<T, RowOp::kResidualIS, VPT, G, S, CSM>(a);
}

// Row buffers in the ring: one.  Measured on B200 (prefill rows, H = 4096):
// deeper rings cost occupancy and lose to more resident CTAs.
template <RowOp OP>
constexpr int stages() { return 1; }

// Constants (gain, cos/sin) in shared memory: holding them in registers
// (8 to 24 floats per slot) costs resident CTAs and rows in flight - measured
// at prefill sizes on B200.
template <RowOp OP>
constexpr bool const_in_smem() { return true; }

template <typename T, RowOp OP, int VPT, bool G>
constexpr auto row_kernel() {
    constexpr int S = stages<OP>();
    constexpr bool C = const_in_smem<OP>();
    if constexpr (OP == RowOp::kRms) return rms_norm_regs_kernel<T, VPT, G, S, C>;
    else if constexpr (OP == RowOp::kInputScale) return input_scale_norm_regs_kernel<T, VPT, G, S, C>;
    else if constexpr (OP == RowOp::kNormGate) return output_norm_gate_row_regs_kernel<T, VPT, G, S, C>;
    else if constexpr (OP == RowOp::kResidual) return norm_residual_regs_kernel<T, VPT, G, S, C>;
    else return norm_residual_input_scale_regs_kernel<T, VPT, G, S, C>;
}

template <typename T, RowOp OP, int VPT, bool G>
cudaError_t launch_row_g(const RowArgs& a0, int nvec, cudaStream_t s) {
    RowArgs a = a0;
    const int nt = ((nvec + VPT - 1) / VPT + 31) / 32 * 32;
    a.rows_per_cta = is_residual(OP) ? kResidualChunk : kRowChunk;
    auto kern = row_kernel<T, OP, VPT, G>();
    const size_t smem = const_in_smem<OP>() ? (size_t)16 * nt * VPT * const_pieces_per_slot<T, OP, G>() : 0;
    if (smem > 32 * 1024) {  // above the default 48 KB once the static part is added
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const int64_t grid = (a.rows + a.rows_per_cta - 1) / a.rows_per_cta;
    return launch_pdl(kern, (unsigned)grid, (unsigned)nt, smem, s, a);
}

template <typename T, RowOp OP, int VPT>
cudaError_t launch_row_vpt(const RowArgs& a, int nvec, cudaStream_t s) {
    return a.gain ? launch_row_g<T, OP, VPT, true>(a, nvec, s) : launch_row_g<T, OP, VPT, false>(a, nvec, s);
}

// Slots per thread: the fewest that fit a row into kThreadsRow threads (small
// CTAs, many resident; twice that for core 5).
constexpr int kThreadsRow = 128;

template <typename T, RowOp OP>
cudaError_t launch_row_t(const RowArgs& a, cudaStream_t s) {
    const int nvec = a.width / Vec<T>::N;
    const int cap = is_residual(OP) ? 2 * kThreadsRow : kThreadsRow;
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
        default: break;  // the fused residual + pre-norm has no register-staged form
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_row_regs(int dtype, RowOp op, const RowArgs& a, cudaStream_t s) {
    return dtype == 0 ? launch_row_dt<__nv_bfloat16>(op, a, s) : launch_row_dt<float>(op, a, s);
}

}  // namespace muse
