// Row-wide normalisation kernels (cores 1, 2, 5 and core 4 with one norm per
// token) on a TMA bulk-copy pipeline.
//
// The rows are dealt round-robin to the CTAs.  One producer warp streams whole
// rows (activation row, plus the gate row for core 4 or the FP32 stream row
// for core 5) from global memory into a ring of S shared-memory stages with
// cp.async.bulk, each stage tracked by a "full" mbarrier (transaction bytes)
// and an "empty" mbarrier (one arrival per consumer warp).  The consumer warps
// read their 16-byte pieces of a stage, release it, reduce the row's sum of
// squares (named barrier among consumers only), and write the outputs.  Rows
// in flight per SM are set by the stage count, not by registers.
//
// Per-expert core 1 (rows grouped by expert) deals each CTA a contiguous run
// of rows instead, and stages expert gain rows through one or two shared slots
// outside the ring: the producer loads a gain row once per change of expert
// (after the consumers have released the slot), each stage carries the index
// of the expert run its row belongs to, and the consumers copy a run's gain to
// registers at its first row.
//
// Every mbarrier wait is bounded: after kSpinLimit polls the thread records a
// timeout in a device-wide error word (read by muse_device_error), stops, and
// the producer waits - again bounded - for its own copies still in flight
// before the CTA exits.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace muse {

__device__ unsigned int g_device_error;  // bit 0: an mbarrier wait timed out

}  // namespace muse

#include "tma_pipe.cuh"

namespace muse {
namespace {

using namespace pipe;

__host__ __device__ constexpr bool t_is_residual(RowOp op) {
    return op == RowOp::kResidual || op == RowOp::kResidualIS || op == RowOp::kResidualPre ||
           op == RowOp::kResidualISPre || op == RowOp::kBlendPre;
}
// _residual_core fused with the next pre-norm: core 5's fused pipeline with
// the branch entering the blend as it is (no branch norm, no cast).
__host__ __device__ constexpr bool t_blend(RowOp op) { return op == RowOp::kBlendPre; }
__host__ __device__ constexpr bool t_scales_first(RowOp op) {
    return op == RowOp::kInputScale || op == RowOp::kResidualIS || op == RowOp::kResidualISPre;
}
__host__ __device__ constexpr bool t_prenorm(RowOp op) {
    return op == RowOp::kResidualPre || op == RowOp::kResidualISPre || op == RowOp::kBlendPre;
}
// Ops whose stage carries the FP32 stream row besides the activation row (core 5).
__host__ __device__ constexpr bool t_f32_row(RowOp op) { return t_is_residual(op); }
// Per-expert core 1: each CTA takes a contiguous run of rows, so consecutive
// rows mostly share an expert, and stages expert gain rows through one or two
// shared slots outside the ring, one load per change of expert; the consumers
// keep the current expert's gain in registers, as core 1 keeps its gain.
__host__ __device__ constexpr bool t_grouped(RowOp op) { return op == RowOp::kRmsGrouped; }
constexpr int kGainSlots = 2;
// Two slots (the next expert's gain can land before the consumers reach it)
// while the CTA's shared memory stays within a quarter of an SM's; else one,
// which keeps four CTAs per SM.
__host__ __device__ inline int grouped_gain_slots(uint32_t ring_bytes, uint32_t gslot_bytes) {
    return ring_bytes + 2u * gslot_bytes <= 48u * 1024u ? 2 : 1;
}

template <typename T, RowOp OP>
struct TmaShape {
    static constexpr int V = Vec<T>::N;
    static constexpr int SV = V / 4;
};

// Byte offsets of one stage: activation row, then gate row (core 4) or FP32
// stream row (core 5), each 128-byte aligned.
struct StageLayout {
    uint32_t x_bytes, x_off, g_off, h_off, stage_bytes;
};

__host__ __device__ inline uint32_t align128(uint32_t v) { return (v + 127u) & ~127u; }

template <typename T, RowOp OP>
__host__ __device__ inline StageLayout stage_layout(int width) {
    StageLayout L;
    L.x_bytes = (uint32_t)width * sizeof(T);
    L.x_off = 0;
    uint32_t off = align128(L.x_bytes);
    L.g_off = off;
    if (OP == RowOp::kNormGate) off += align128(L.x_bytes);
    L.h_off = off;
    if (t_f32_row(OP)) off += align128((uint32_t)width * 4u);
    L.stage_bytes = off;
    return L;
}

template <typename T, RowOp OP, int VPT, bool HAS_GAIN, int S>
__device__ __forceinline__ void row_tma_body(const RowArgs& a) {
    using Sh = TmaShape<T, OP>;
    constexpr int V = Sh::V, SV = Sh::SV;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ float red[2][32];
    __shared__ __align__(8) uint64_t full_bar[S];
    __shared__ __align__(8) uint64_t empty_bar[S];
    // per-expert core 1: with N slots, slot j holds expert runs j, j + N, ...
    // of this CTA's rows; full completes when a run's gain row has landed,
    // free when every consumer warp has copied it to registers; stage_run[s]
    // is the run of the row in stage s (written before the stage's full arrive)
    __shared__ __align__(8) uint64_t gain_full[t_grouped(OP) ? kGainSlots : 1];
    __shared__ __align__(8) uint64_t gain_free[t_grouped(OP) ? kGainSlots : 1];
    __shared__ int stage_run[t_grouped(OP) ? S : 1];

    const int ncons = blockDim.x - 32;  // consumer threads; the last warp produces
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int nvec = a.width / V;
    const StageLayout L = stage_layout<T, OP>(a.width);
    const uint32_t lim = a.spin_limit ? a.spin_limit : kSpinLimit;  // polls per mbarrier wait

    // This CTA's rows: r0, r0 + step, ... - rows interleaved across the grid,
    // so at any time the CTAs stream one compact window of the tensors
    // (measured slightly ahead of contiguous chunks per CTA when the previous
    // kernel left dirty lines in L2); per-expert core 1 takes a contiguous run.
    const int64_t step = t_grouped(OP) ? 1 : gridDim.x;
    const int64_t r0 = t_grouped(OP) ? (int64_t)blockIdx.x * a.rows / gridDim.x : (int64_t)blockIdx.x;
    const int n = t_grouped(OP) ? (int)(((int64_t)blockIdx.x + 1) * a.rows / gridDim.x - r0)
                                : (int)max((int64_t)0, (a.rows - r0 + step - 1) / step);
    // the expert gain slots, after the ring
    const uint32_t gslot_bytes = align128((uint32_t)a.width * 4u);
    unsigned char* gslots = smem + (size_t)S * L.stage_bytes;
    const int nslots = grouped_gain_slots((uint32_t)S * L.stage_bytes, gslot_bytes);

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], (uint32_t)(ncons >> 5));
        }
        if constexpr (t_grouped(OP)) {
            for (int j = 0; j < kGainSlots; ++j) {
                mbar_init(&gain_full[j], 1);
                mbar_init(&gain_free[j], (uint32_t)(ncons >> 5));
            }
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp == (ncons >> 5)) {
        // ---------------- producer warp: lane 0 issues whole-row bulk copies
        // per-expert core 1: the first row's group (the last g with
        // offsets[g] <= row), found by the whole warp with 32 probes a round;
        // every index read stays in [0, num_groups - 1] whatever the table holds
        int g_first = 0;
        if constexpr (t_grouped(OP)) {
            if (n > 0) {
                int lo = 0, hi = a.num_groups;
                while (hi - lo > 1) {
                    const int chunk = (hi - lo + 31) >> 5;
                    const int probe = lo + lane * chunk;
                    const bool le = probe < hi && (int64_t)__ldg(a.group_offsets + probe) <= r0;
                    const unsigned m = __ballot_sync(0xffffffffu, le);
                    const int last = m ? 31 - __clz(m) : 0;
                    const int nlo = lo + last * chunk;
                    hi = min(hi, nlo + chunk);
                    lo = nlo;
                }
                g_first = lo;
            }
        }
        if (lane == 0) {
            uint32_t bytes = L.x_bytes;
            if (OP == RowOp::kNormGate) bytes += L.x_bytes;
            if (t_f32_row(OP)) bytes += (uint32_t)a.width * 4u;
            int issued = 0;
            bool ok = true;
            int grp = -1, runs = 0;  // per-expert core 1: current group, runs started
            for (int k = 0; k < n && ok; ++k) {
                const int s = k % S;
                const int64_t row = r0 + k * step;
                // bounded-wait probe: this row's stage is never signalled
                if (a.probe_stall && row == a.stall_row) break;
                if (k >= S) ok = mbar_wait(&empty_bar[s], (uint32_t)((k / S - 1) & 1), lim);
                if (!ok) break;
                unsigned char* st = smem + (size_t)s * L.stage_bytes;
                if constexpr (t_grouped(OP)) {
                    // the activation copy first; the stage's run index is written
                    // before the producer's arrival, which completes the phase
                    mbar_expect_tx(&full_bar[s], bytes);
                    bulk_g2s(st + L.x_off, static_cast<const char*>(a.x) + row * a.x_stride * (int64_t)sizeof(T),
                             L.x_bytes, &full_bar[s]);
                    // the row's group: the first row's, then a forward walk
                    int g = g_first;
                    if (grp >= 0) {
                        g = grp;
                        while (g + 1 < a.num_groups && (int64_t)__ldg(a.group_offsets + g + 1) <= row) ++g;
                    }
                    if (g != grp) {
                        // a new run: its slot's previous run must be released first
                        const int j = runs % nslots;
                        if (runs >= nslots) ok = mbar_wait(&gain_free[j], (uint32_t)((runs / nslots - 1) & 1), lim);
                        if (ok) {
                            mbar_arrive_expect_tx(&gain_full[j], (uint32_t)a.width * 4u);
                            bulk_g2s(gslots + (size_t)j * gslot_bytes, a.gain + (int64_t)g * a.width,
                                     (uint32_t)a.width * 4u, &gain_full[j]);
                            grp = g;
                            ++runs;
                        }
                    }
                    stage_run[s] = runs - 1;
                    // arrive even after a timed-out wait: the activation copy is
                    // in flight and the exit waits below must see it land
                    mbar_arrive(&full_bar[s]);
                    ++issued;
                    continue;
                }
                mbar_arrive_expect_tx(&full_bar[s], bytes);
                bulk_g2s(st + L.x_off, static_cast<const char*>(a.x) + row * a.x_stride * (int64_t)sizeof(T),
                         L.x_bytes, &full_bar[s]);
                if constexpr (OP == RowOp::kNormGate)
                    bulk_g2s(st + L.g_off, static_cast<const char*>(a.gate) + row * a.gate_stride * (int64_t)sizeof(T),
                             L.x_bytes, &full_bar[s]);
                if constexpr (t_is_residual(OP))
                    bulk_g2s(st + L.h_off, a.stream_in + row * a.s_in_stride, (uint32_t)a.width * 4u, &full_bar[s]);
                ++issued;
            }
            // Before exiting, every copy this CTA issued must have landed: in
            // the normal path the consumers already waited on them, so these
            // waits return at once.
            for (int k = max(0, issued - S); k < issued; ++k)
                if (!mbar_wait(&full_bar[k % S], (uint32_t)((k / S) & 1), lim)) break;
            if constexpr (t_grouped(OP)) {
                for (int r = max(0, runs - nslots); r < runs; ++r)
                    if (!mbar_wait(&gain_full[r % nslots], (uint32_t)((r / nslots) & 1), lim)) break;
            }
        }
        return;
    }

    // ---------------- consumer warps
    // Element arithmetic on packed FP32 pairs (f32x2: two IEEE round-to-nearest
    // operations per instruction); offsets and the stage walk are incremental.
    constexpr int P = V / 2;
    bool valid[VPT];
    uint32_t voff[VPT];  // this thread's byte offset of slot i within a row
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        valid[i] = tid + i * ncons < nvec;
        voff[i] = (uint32_t)(tid + i * ncons) * 16u;
    }

    // per-slot constants in registers (the pipeline, not registers, holds the
    // rows in flight): effective gain, cos and sin of the blend angle
    f32x2 w[HAS_GAIN ? VPT : 1][P];
    f32x2 cth[t_is_residual(OP) ? VPT : 1][P];
    f32x2 sth[t_is_residual(OP) ? VPT : 1][P];
    {
        const f32x2 off2 = f2_make(a.gain_offset, a.gain_offset);
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = valid[i] ? tid + i * ncons : 0;
#pragma unroll
            for (int k = 0; k < SV; ++k) {
                if constexpr (HAS_GAIN && OP != RowOp::kRmsGrouped) {
                    const float4 g4 = __ldg(reinterpret_cast<const float4*>(a.gain) + v * SV + k);
                    w[i][2 * k] = f2_add(f2_make(g4.x, g4.y), off2);  // FP32 sums
                    w[i][2 * k + 1] = f2_add(f2_make(g4.z, g4.w), off2);
                }
                if constexpr (t_is_residual(OP)) {
                    const float4 t4 = __ldg(reinterpret_cast<const float4*>(a.theta) + v * SV + k);
                    float s0, c0, s1, c1, s2, c2, s3, c3;
                    sincosf(t4.x, &s0, &c0);
                    sincosf(t4.y, &s1, &c1);
                    sincosf(t4.z, &s2, &c2);
                    sincosf(t4.w, &s3, &c3);
                    cth[i][2 * k] = f2_make(c0, c1);
                    cth[i][2 * k + 1] = f2_make(c2, c3);
                    sth[i][2 * k] = f2_make(s0, s1);
                    sth[i][2 * k + 1] = f2_make(s2, s3);
                }
            }
        }
    }
    const float inv_width = 1.0f / (float)a.width;

    // output row pointer, advanced one row per iteration
    char* out_row = t_is_residual(OP)
        ? reinterpret_cast<char*>(a.stream_out + r0 * a.s_out_stride)
        : static_cast<char*>(a.y) + r0 * a.y_stride * (int64_t)sizeof(T);
    const int64_t out_step = step * (t_is_residual(OP) ? a.s_out_stride * (int64_t)sizeof(float)
                                                      : a.y_stride * (int64_t)sizeof(T));
    // fused ops: the next sublayer's effective gain in shared memory, after the
    // ring (written here, first read after the row's first consumer barrier)
    float* w2s = reinterpret_cast<float*>(smem + (size_t)S * L.stage_bytes);
    if constexpr (t_prenorm(OP)) {
        if (a.gain2)
            for (int j = tid; j < a.width; j += ncons) w2s[j] = __ldg(a.gain2 + j) + a.gain2_offset;  // FP32 sum
    }
    // pre-norm output rows (fused ops only)
    const int64_t y_es = a.y_f32 ? 4 : (int64_t)sizeof(T);
    char* y_row = t_prenorm(OP) ? static_cast<char*>(a.y) + r0 * a.y_stride * y_es : nullptr;
    const int64_t y_step = step * a.y_stride * y_es;

    // After a timed-out wait a warp stops touching the ring and the outputs but
    // keeps joining the consumer barrier, so no other warp is left waiting.
    bool alive = true;
    int bank = 0;
    int s = 0;
    uint32_t phase = 0;
    int run = -1;  // per-expert core 1: the expert run whose gain slot this warp holds
    for (int k = 0; k < n; ++k) {
        if (alive) alive = mbar_wait(&full_bar[s], phase, lim);
        alive = __all_sync(0xffffffffu, alive);
        const unsigned char* st = smem + s * L.stage_bytes;
        if constexpr (t_grouped(OP)) {
            const int r = alive ? stage_run[s] : run;
            if (r != run && alive) {
                // the first row of the next expert run: wait for its gain row,
                // copy it (plus the offset, an FP32 sum) to registers, release the slot
                run = r;
                alive = mbar_wait(&gain_full[run % nslots], (uint32_t)((run / nslots) & 1), lim);
                alive = __all_sync(0xffffffffu, alive);
                if (alive) {
                    if constexpr (HAS_GAIN) {
                        const unsigned char* gs = gslots + (size_t)(run % nslots) * gslot_bytes;
                        const f32x2 off2 = f2_make(a.gain_offset, a.gain_offset);
#pragma unroll
                        for (int i = 0; i < VPT; ++i) {
                            if (!valid[i]) continue;
#pragma unroll
                            for (int q = 0; q < SV; ++q) {
                                const float4 g4 = *reinterpret_cast<const float4*>(gs + voff[i] * SV + 16u * q);
                                w[i][2 * q] = f2_add(f2_make(g4.x, g4.y), off2);
                                w[i][2 * q + 1] = f2_add(f2_make(g4.z, g4.w), off2);
                            }
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&gain_free[run % nslots]);
                }
            }
        }
        uint4 xv[VPT], gv[OP == RowOp::kNormGate ? VPT : 1], hv[t_f32_row(OP) ? VPT * SV : 1];
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const bool rd = alive && valid[i];
            xv[i] = rd ? *reinterpret_cast<const uint4*>(st + L.x_off + voff[i]) : make_uint4(0, 0, 0, 0);
            if constexpr (OP == RowOp::kNormGate)
                gv[i] = rd ? *reinterpret_cast<const uint4*>(st + L.g_off + voff[i]) : make_uint4(0, 0, 0, 0);
            if constexpr (t_f32_row(OP)) {
#pragma unroll
                for (int q = 0; q < SV; ++q)
                    hv[i * SV + q] = rd ? *reinterpret_cast<const uint4*>(st + L.h_off + voff[i] * SV + 16u * q)
                                        : make_uint4(0, 0, 0, 0);
            }
        }
        // this warp is done with the stage
        __syncwarp();
        if (lane == 0 && alive) mbar_arrive(&empty_bar[s]);
        if (++s == S) {
            s = 0;
            phase ^= 1u;
        }

        f32x2 x[VPT][P];
        f32x2 acc[2] = {f2_make(0.0f, 0.0f), f2_make(0.0f, 0.0f)};  // 4 partial sums
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            to_pairs<T>(xv[i], x[i]);
#pragma unroll
            for (int q = 0; q < P; ++q) {
                if constexpr (t_scales_first(OP) && HAS_GAIN) x[i][q] = f2_mul(x[i][q], w[i][q]);
                acc[q & 1] = f2_fma(x[i][q], x[i][q], acc[q & 1]);
            }
        }
        float r = 1.0f;
        if constexpr (!t_blend(OP)) {  // the branch norm (the blend alone has none)
            const float part = f2_sum(acc[0]) + f2_sum(acc[1]);
            r = inv_rms_fast(consumer_sum(part, red, bank, ncons), inv_width, a.eps);
        }
        const f32x2 r2 = f2_make(r, r);

        if constexpr (OP == RowOp::kRms || OP == RowOp::kInputScale || OP == RowOp::kNormGate ||
                      OP == RowOp::kRmsGrouped) {
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                f32x2 o[P];
#pragma unroll
                for (int q = 0; q < P; ++q) {
                    o[q] = f2_mul(x[i][q], r2);
                    if constexpr ((OP == RowOp::kRms || OP == RowOp::kRmsGrouped) && HAS_GAIN)
                        o[q] = f2_mul(o[q], w[i][q]);
                }
                if constexpr (OP == RowOp::kNormGate) {
                    float gf[V];
                    unpack<T>(gv[i], gf);
#pragma unroll
                    for (int q = 0; q < P; ++q) {
                        float lo, hi;
                        f2_split(o[q], lo, hi);
                        o[q] = f2_make(times_sigmoid<T>(lo, gf[2 * q]), times_sigmoid<T>(hi, gf[2 * q + 1]));
                    }
                }
                if (alive && valid[i]) st_vec(out_row + voff[i], from_pairs<T>(o));
            }
        } else {
            f32x2 hs[t_prenorm(OP) ? VPT : 1][P];  // the new stream, for the pre-norm
            f32x2 hss = f2_make(0.0f, 0.0f);
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                f32x2 h[P], o[P];
#pragma unroll
                for (int q = 0; q < SV; ++q) to_pairs<float>(hv[i * SV + q], h + 2 * q);
#pragma unroll
                for (int q = 0; q < P; ++q) {
                    f32x2 t = f2_mul(x[i][q], r2);  // z r when the gain came first
                    if constexpr (!t_scales_first(OP) && HAS_GAIN) t = f2_mul(t, w[i][q]);
                    // cast back to the branch dtype; the blend alone takes the branch as read
                    const f32x2 nb = t_blend(OP) ? x[i][q] : round_pair<T>(t);
                    o[q] = f2_fma(cth[i][q], h[q], f2_mul(sth[i][q], nb));
                    if constexpr (t_prenorm(OP)) {
                        hs[i][q] = o[q];
                        hss = f2_fma(o[q], o[q], hss);
                    }
                }
                if (alive && valid[i]) {
#pragma unroll
                    for (int q = 0; q < SV; ++q) st_vec(out_row + voff[i] * SV + 16u * q, from_pairs<float>(o + 2 * q));
                }
            }
            if constexpr (t_prenorm(OP)) {
                // next sublayer's pre-norm of the new FP32 stream: y = (h' r(h')) w2,
                // cast once; w2 from shared memory (filled once per CTA)
                const float rr = inv_rms_fast(consumer_sum(f2_sum(hss), red, bank, ncons), inv_width, a.eps2);
                const f32x2 rr2 = f2_make(rr, rr);
#pragma unroll
                for (int i = 0; i < VPT; ++i) {
                    f32x2 y[P];
                    const int wi = valid[i] ? (int)(voff[i] >> 4) * V : 0;  // idle slots read column 0
#pragma unroll
                    for (int q = 0; q < P; ++q) {
                        y[q] = f2_mul(hs[i][q], rr2);
                        if (a.gain2) y[q] = f2_mul(y[q], *reinterpret_cast<const f32x2*>(w2s + wi + 2 * q));
                    }
                    if (alive && valid[i]) {
                        if (a.y_f32) {
#pragma unroll
                            for (int q = 0; q < SV; ++q) st_vec(y_row + voff[i] * SV + 16u * q, from_pairs<float>(y + 2 * q));
                        } else {
                            st_vec(y_row + voff[i], from_pairs<T>(y));
                        }
                    }
                }
                y_row += y_step;
            }
        }
        out_row += out_step;
    }
}

// One entry symbol per core, so launch lists and profiles name the core.
// Cores 1, 2, 4 and per-expert core 1 use at most 256 consumers (288 threads)
// and keep a register budget for four resident CTAs up to two slots per
// thread (two at four slots); core 5's one-slot instances (up to 544 threads)
// keep one for two resident CTAs.  One CTA fewer per SM measured 8-20% slower.
constexpr int kRowThreads = 256 + 32;
template <typename T, int VPT, bool G, int S>
__global__ void __launch_bounds__(kRowThreads, VPT <= 2 ? 4 : 2) rms_norm_kernel(const __grid_constant__ RowArgs a) {
    pdl_begin();
    row_tma_body<T, RowOp::kRms, VPT, G, S>(a);
}
template <typename T, int VPT, bool G, int S>
__global__ void __launch_bounds__(kRowThreads, VPT <= 2 ? 4 : 2) input_scale_norm_kernel(const __grid_constant__ RowArgs a) {
    pdl_begin();
    row_tma_body<T, RowOp::kInputScale, VPT, G, S>(a);
}
template <typename T, int VPT, bool G, int S>
__global__ void __launch_bounds__(kRowThreads, VPT <= 2 ? 4 : 2) output_norm_gate_row_kernel(const __grid_constant__ RowArgs a) {
    pdl_begin();
    row_tma_body<T, RowOp::kNormGate, VPT, G, S>(a);
}
template <typename T, int VPT, bool G, int S>
__global__ void __launch_bounds__(512 + 32, VPT == 1 ? 2 : 1) norm_residual_kernel(const __grid_constant__ RowArgs a) {
    pdl_begin();
    row_tma_body<T, RowOp::kResidual, VPT, G, S>(a);
}
template <typename T, int VPT, bool G, int S>
__global__ void __launch_bounds__(512 + 32, VPT == 1 ? 2 : 1) norm_residual_input_scale_kernel(const __grid_constant__ RowArgs a) {
    pdl_begin();
    row_tma_body<T, RowOp::kResidualIS, VPT, G, S>(a);
}
template <typename T, int VPT, bool G, int S>
__global__ void __launch_bounds__(kRowThreads, VPT <= 2 ? 4 : 2) rms_norm_grouped_kernel(const __grid_constant__ RowArgs a) {
    pdl_begin();
    row_tma_body<T, RowOp::kRmsGrouped, VPT, G, S>(a);
}
template <typename T, int VPT, bool G, int S>
__global__ void __launch_bounds__(512 + 32, VPT == 1 ? 2 : 1) norm_residual_prenorm_kernel(const __grid_constant__ RowArgs a) {
    pdl_begin();
    row_tma_body<T, RowOp::kResidualPre, VPT, G, S>(a);
}
template <typename T, int VPT, bool G, int S>
__global__ void __launch_bounds__(512 + 32, VPT == 1 ? 2 : 1) norm_residual_input_scale_prenorm_kernel(const __grid_constant__ RowArgs a) {
    pdl_begin();
    row_tma_body<T, RowOp::kResidualISPre, VPT, G, S>(a);
}

template <typename T, int VPT, bool G, int S>
__global__ void __launch_bounds__(512 + 32, VPT == 1 ? 2 : 1) residual_blend_prenorm_kernel(const __grid_constant__ RowArgs a) {
    pdl_begin();
    row_tma_body<T, RowOp::kBlendPre, VPT, G, S>(a);
}

template <typename T, RowOp OP, int VPT, bool G, int S>
constexpr auto row_tma_kernel() {
    if constexpr (OP == RowOp::kRms) return rms_norm_kernel<T, VPT, G, S>;
    else if constexpr (OP == RowOp::kInputScale) return input_scale_norm_kernel<T, VPT, G, S>;
    else if constexpr (OP == RowOp::kNormGate) return output_norm_gate_row_kernel<T, VPT, G, S>;
    else if constexpr (OP == RowOp::kResidual) return norm_residual_kernel<T, VPT, G, S>;
    else if constexpr (OP == RowOp::kResidualIS) return norm_residual_input_scale_kernel<T, VPT, G, S>;
    else if constexpr (OP == RowOp::kResidualPre) return norm_residual_prenorm_kernel<T, VPT, G, S>;
    else if constexpr (OP == RowOp::kRmsGrouped) return rms_norm_grouped_kernel<T, VPT, G, S>;
    else if constexpr (OP == RowOp::kBlendPre) return residual_blend_prenorm_kernel<T, VPT, G, S>;
    else return norm_residual_input_scale_prenorm_kernel<T, VPT, G, S>;
}

}  // namespace

// Stage count and consumer threads per op; launch shape.
template <typename T, RowOp OP, int VPT, bool G, int S>
cudaError_t launch_row_tma_s(const RowArgs& a0, int nvec, cudaStream_t s) {
    RowArgs a = a0;
    const int ncons = ((nvec + VPT - 1) / VPT + 31) / 32 * 32;
    const int threads = ncons + 32;
    const StageLayout L = stage_layout<T, OP>(a.width);
    const uint32_t gslot = align128((uint32_t)a.width * 4u);
    const size_t smem = (size_t)S * L.stage_bytes + (t_prenorm(OP) ? (size_t)a.width * 4 : 0) +
                        (t_grouped(OP) ? (size_t)grouped_gain_slots((uint32_t)S * L.stage_bytes, gslot) * gslot : 0);
    auto kern = row_tma_kernel<T, OP, VPT, G, S>();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int per_sm = blocks_per_sm((const void*)kern, threads, smem);
    int64_t grid = (int64_t)per_sm * sm_count();
    if (grid > a.rows) grid = a.rows;
    if (grid < 1) grid = 1;
    return launch_pdl(kern, (unsigned)grid, (unsigned)threads, smem, s, a);
}

template <typename T, RowOp OP, int VPT, bool G>
cudaError_t launch_row_tma_v(const RowArgs& a, int nvec, int stages, cudaStream_t s) {
    if (stages >= 3) return launch_row_tma_s<T, OP, VPT, G, 3>(a, nvec, s);
    return launch_row_tma_s<T, OP, VPT, G, 2>(a, nvec, s);
}

// Launch shape, measured on B200 at prefill sizes (H = 4096): two or three
// stages per CTA and as many CTAs per SM as fit beat deeper rings (4 CTAs of
// 256 consumers for 8 KB rows; 2 CTAs of 512 consumers, one slot each, for
// core 5's 24 KB rows - ahead of 256 consumers x 2 slots inside the five-core
// step).  Core 5 keeps at most 2 slots per consumer thread (its 24 per-slot
// constants live in registers).
constexpr uint32_t kRingMaxBytes = 200 * 1024;
constexpr int kConsumers = 256;
static_assert(kRowThreads == kConsumers + 32, "launch bounds of the non-residual row kernels");

template <typename T, RowOp OP>
cudaError_t launch_row_op(const RowArgs& a, cudaStream_t s) {
    const int nvec = a.width / Vec<T>::N;
    const StageLayout L = stage_layout<T, OP>(a.width);
    const int dt = std::is_same<T, float>::value ? 1 : 0;
    if (2 * L.stage_bytes > kRingMaxBytes) {
        if constexpr (t_prenorm(OP) || OP == RowOp::kRmsGrouped) return cudaErrorInvalidValue;  // the API keeps these rows in range
        return launch_row_regs(dt, OP, a, s);
    }
    const int stages = L.stage_bytes >= 16 * 1024 ? 2 : 3;
    const bool g = a.gain != nullptr;
    // slots per consumer thread: the fewest that fit a row into kConsumers
    // threads (core 5: at most 2 slots, up to twice the consumers)
    if (nvec <= kConsumers || (t_is_residual(OP) && nvec <= 2 * kConsumers))
        return g ? launch_row_tma_v<T, OP, 1, true>(a, nvec, stages, s) : launch_row_tma_v<T, OP, 1, false>(a, nvec, stages, s);
    if (nvec <= 2 * kConsumers || (t_is_residual(OP) && nvec <= 4 * kConsumers))
        return g ? launch_row_tma_v<T, OP, 2, true>(a, nvec, stages, s) : launch_row_tma_v<T, OP, 2, false>(a, nvec, stages, s);
    if constexpr (!t_is_residual(OP)) {
        if (nvec <= 4 * kConsumers)
            return g ? launch_row_tma_v<T, OP, 4, true>(a, nvec, stages, s) : launch_row_tma_v<T, OP, 4, false>(a, nvec, stages, s);
    }
    if constexpr (t_prenorm(OP) || OP == RowOp::kRmsGrouped) return cudaErrorInvalidValue;
    return launch_row_regs(dt, OP, a, s);
}

template <typename T>
cudaError_t launch_row_t2(RowOp op, const RowArgs& a, cudaStream_t s) {
    switch (op) {
        case RowOp::kRms: return launch_row_op<T, RowOp::kRms>(a, s);
        case RowOp::kInputScale: return launch_row_op<T, RowOp::kInputScale>(a, s);
        case RowOp::kNormGate: return launch_row_op<T, RowOp::kNormGate>(a, s);
        case RowOp::kResidual: return launch_row_op<T, RowOp::kResidual>(a, s);
        case RowOp::kResidualIS: return launch_row_op<T, RowOp::kResidualIS>(a, s);
        case RowOp::kResidualPre: return launch_row_op<T, RowOp::kResidualPre>(a, s);
        case RowOp::kResidualISPre: return launch_row_op<T, RowOp::kResidualISPre>(a, s);
        case RowOp::kRmsGrouped: return launch_row_op<T, RowOp::kRmsGrouped>(a, s);
        case RowOp::kBlendPre: return launch_row_op<T, RowOp::kBlendPre>(a, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_row(int dtype, RowOp op, const RowArgs& a, cudaStream_t s) {
    return dtype == 0 ? launch_row_t2<__nv_bfloat16>(op, a, s) : launch_row_t2<float>(op, a, s);
}

cudaError_t read_device_error(unsigned int* out, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_device_error, sizeof(unsigned int));
    if (e != cudaSuccess || !clear) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned int));
}

}  // namespace muse

