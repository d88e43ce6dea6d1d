// Backward of the row-wide cores: core 1 (_rms_norm_core), core 2
// (_input_scale_norm_core) and core 5 (_norm_residual_core with the
// per-channel cos/sin blend).  The cores run under autograd, so the backward
// is the derivative of each forward map, evaluated from the saved forward
// inputs with r recomputed; every dtype boundary the forward materialises
// passes the gradient back rounded to that tensor's dtype.
//
//   core 1:  g = dy w;  dx = r g - r^3 x (sum_j g_j x_j) / H;
//            dgain += dy x r
//   core 2:  z = x w;  dz = r dy - r^3 z (sum_j dy_j z_j) / H;
//            dx = dz w;  dgain += dz x
//   core 5:  dh = cos(theta) dh';  dnb = cast_branch(sin(theta) dh');
//            dbranch = the core 1 (or core 2) form applied to dnb;
//            dtheta += dh' (-sin(theta) h + cos(theta) nb), nb the forward's
//            cast branch
//
// Same pipeline as the forward row kernels (row_tma.cu): a producer warp
// streams each row's inputs (x and dy; core 5: branch, dh' and h) into a ring
// of shared-memory stages with cp.async.bulk; the consumer warps reduce the
// row's two sums (sum of squares and the gradient dot product) with one
// named barrier and write the input gradients.  The rows are dealt
// round-robin to a persistent grid; each consumer thread owns the same
// columns in every row, so it accumulates its columns' gain / theta
// gradients in registers and writes one partial row per CTA into the
// caller's workspace, which a second kernel sums in a fixed order.
//
// Core 5 rows of more than 512 16-byte vectors (up to 1024) are split over a
// cluster of CL CTAs: each CTA streams and owns one CL-th of every row's
// columns (one slot per consumer thread, as for narrower rows), and the CTAs
// swap their parts' row sums through distributed shared memory (per row, an
// asynchronous store into each peer that completes transaction bytes on the
// peer's mbarrier); every CTA adds the parts in rank order, so all use the
// same r.  Holding two slots of per-column constants and accumulators per
// thread instead spilled registers and ran at a third of the bandwidth.
#include <map>
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace muse {
namespace {
__device__ unsigned int g_device_error;  // nonzero: an mbarrier wait of the row backward timed out
}  // namespace
}  // namespace muse

#include "tma_pipe.cuh"

namespace muse {
namespace {

using namespace pipe;

__host__ __device__ constexpr bool b_is_res(BwdOp op) { return op == BwdOp::kResidual || op == BwdOp::kResidualIS; }
__host__ __device__ constexpr bool b_gain_first(BwdOp op) { return op == BwdOp::kInputScale || op == BwdOp::kResidualIS; }

// At most this many resident CTAs per SM (bounds the workspace).
constexpr int kBwdMaxCtasPerSm = 4;
// CTAs per cluster for core 5 rows of more than 512 vectors (two when the
// vector count does not divide by four).  Measured on B200 (32768 rows of
// 8192 / 80251 rows of 5120), launched back to back / alone: four CTAs 716 /
// 695 and 1204 / 1158 us, two CTAs 776 / 765 and 1453 / 1433 us.  Cluster
// launches go without programmatic dependent launch: with it, four-CTA
// clusters launched back to back took 1285 / 1815 us.
constexpr int kSplitCtas = 4;

__host__ __device__ inline uint32_t al128(uint32_t v) { return (v + 127u) & ~127u; }

struct BwdLayout {
    uint32_t x_bytes, dy_bytes, h_bytes, dy_off, h_off, stage_bytes;
};

template <typename T, BwdOp OP>
__host__ __device__ inline BwdLayout bwd_layout(int width) {
    BwdLayout L;
    L.x_bytes = (uint32_t)width * sizeof(T);
    L.dy_bytes = (uint32_t)width * (b_is_res(OP) ? 4u : (uint32_t)sizeof(T));
    L.h_bytes = b_is_res(OP) ? (uint32_t)width * 4u : 0u;
    L.dy_off = al128(L.x_bytes);
    L.h_off = L.dy_off + al128(L.dy_bytes);
    L.stage_bytes = L.h_off + al128(L.h_bytes);
    return L;
}

// ---- clusters of CTAs that split core 5 rows
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Every thread of every CTA of the cluster arrives, then waits (release / acquire).
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
// Shared address of the same variable in the CTA of the given cluster rank.
__device__ __forceinline__ uint32_t peer_addr(const void* p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
    return r;
}
// Two floats into the peer's shared memory by an asynchronous store that
// completes 8 transaction bytes on the peer's mbarrier when they land (the
// peer posts the expected bytes itself; no fence on this side).
__device__ __forceinline__ void push_to_peer(uint32_t val_addr, uint32_t bar_addr, float a, float b) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];"
                 ::"r"(val_addr), "f"(a), "f"(b), "r"(bar_addr) : "memory");
}
// Bounded wait (acquire at cluster scope) for a phase that peers complete.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, uint32_t limit = kSpinLimit) {
    for (uint32_t i = 0; i < limit; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(smem_addr(bar)), "r"(parity)
            : "memory");
        if (done) return true;
    }
    atomicOr(&g_device_error, 1u);
    return false;
}

// Sums of two values over the consumer threads; two banks, one barrier.
__device__ __forceinline__ float2 consumer_sum2(float a, float b, float (*red)[2][32], int& bank, int ncons) {
    a = group_sum<32>(a);
    b = group_sum<32>(b);
    const int nw = ncons >> 5;
    if (nw == 1) return make_float2(a, b);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        red[bank][0][warp] = a;
        red[bank][1][warp] = b;
    }
    consumer_sync(ncons);
    const float ta = lane < nw ? red[bank][0][lane] : 0.0f;
    const float tb = lane < nw ? red[bank][1][lane] : 0.0f;
    bank ^= 1;
    return make_float2(group_sum<32>(ta), group_sum<32>(tb));
}

// 16-byte vector of T at byte offset `off` of a shared stage -> V floats.
template <typename T>
__device__ __forceinline__ void ld_stage(const unsigned char* p, float* f) {
    unpack<T>(*reinterpret_cast<const uint4*>(p), f);
}
// V floats of an FP32 row at element offset e0 of a shared stage.
template <int V>
__device__ __forceinline__ void ld_stage_f32(const unsigned char* p, float* f) {
#pragma unroll
    for (int q = 0; q < V / 4; ++q) {
        const float4 v = *reinterpret_cast<const float4*>(p + 16 * q);
        f[4 * q] = v.x; f[4 * q + 1] = v.y; f[4 * q + 2] = v.z; f[4 * q + 3] = v.w;
    }
}
template <int V>
__device__ __forceinline__ void st_f32(float* p, const float* f) {
#pragma unroll
    for (int q = 0; q < V / 4; ++q)
        *reinterpret_cast<float4*>(p + 4 * q) = make_float4(f[4 * q], f[4 * q + 1], f[4 * q + 2], f[4 * q + 3]);
}

template <typename T, BwdOp OP, int VPT, bool G, int S, int CL>
__device__ __forceinline__ void row_bwd_body(const RowBwdArgs& a) {
    constexpr int V = Vec<T>::N;
    constexpr bool RES = b_is_res(OP);
    constexpr bool FIRST = b_gain_first(OP);
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ float red[2][2][32];
    __shared__ __align__(8) uint64_t full_bar[S];
    __shared__ __align__(8) uint64_t empty_bar[S];
    // CL > 1: xbar[j] completes when every peer's row sums of a row k with
    // k % 2 == j have landed in xval[j][peer rank] (one local arrive that
    // posts the expected bytes, the peers' asynchronous stores complete them)
    constexpr uint32_t kXBytes = 8u * (CL - 1);
    __shared__ __align__(8) uint64_t xbar[2];
    __shared__ __align__(8) float xval[2][CL][2];

    const int ncons = blockDim.x - 32;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    // CL > 1: this CTA owns columns [cbase, cbase + lw) of every row its
    // cluster takes; a cluster takes rows blockIdx.x / CL, + grid / CL, ...
    const uint32_t crank = CL > 1 ? cluster_rank() : 0u;
    const int lw = a.width / CL;
    const int cbase = (int)crank * lw;
    const int nvec = lw / V;
    const BwdLayout L = bwd_layout<T, OP>(lw);
    const int64_t step = gridDim.x / CL;
    const int64_t r0 = blockIdx.x / CL;
    const int n = (int)max((int64_t)0, (a.rows - r0 + step - 1) / step);
    const uint32_t dy_es = RES ? 4u : (uint32_t)sizeof(T);

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], (uint32_t)(ncons >> 5));
        }
        if constexpr (CL > 1) {
            mbar_init(&xbar[0], 1);
            mbar_init(&xbar[1], 1);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        if constexpr (CL > 1) {  // rows 0 and 1
            mbar_arrive_expect_tx(&xbar[0], kXBytes);
            mbar_arrive_expect_tx(&xbar[1], kXBytes);
        }
    }
    __syncthreads();
    // every CTA's barriers are initialised before any peer pushes to it
    if constexpr (CL > 1) cluster_sync_all();

    if (warp == (ncons >> 5)) {
        // ---------------- producer warp: lane 0 issues whole-row bulk copies
        if (lane == 0) {
            const uint32_t bytes = L.x_bytes + L.dy_bytes + L.h_bytes;
            int issued = 0;
            for (int k = 0; k < n; ++k) {
                const int s = k % S;
                if (k >= S && !mbar_wait(&empty_bar[s], (uint32_t)((k / S - 1) & 1))) break;
                unsigned char* st = smem + (size_t)s * L.stage_bytes;
                const int64_t row = r0 + k * step;
                mbar_arrive_expect_tx(&full_bar[s], bytes);
                bulk_g2s(st, static_cast<const char*>(a.x) + (row * a.x_stride + cbase) * (int64_t)sizeof(T),
                         L.x_bytes, &full_bar[s]);
                bulk_g2s(st + L.dy_off, static_cast<const char*>(a.dy) + (row * a.dy_stride + cbase) * (int64_t)dy_es,
                         L.dy_bytes, &full_bar[s]);
                if constexpr (RES)
                    bulk_g2s(st + L.h_off, a.stream_in + row * (int64_t)a.width + cbase, L.h_bytes, &full_bar[s]);
                ++issued;
            }
            for (int k = max(0, issued - S); k < issued; ++k)
                if (!mbar_wait(&full_bar[k % S], (uint32_t)((k / S) & 1))) break;
        }
        if constexpr (CL > 1) cluster_sync_all();  // pairs with the consumers' final one
        return;
    }

    // ---------------- consumer warps: slot i covers vector tid + i * ncons
    bool valid[VPT];
    int col[VPT];   // column within this CTA's part of the row (stage offsets)
    int gcol[VPT];  // column of the row (parameters, outputs)
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        valid[i] = tid + i * ncons < nvec;
        col[i] = valid[i] ? (tid + i * ncons) * V : 0;
        gcol[i] = cbase + col[i];
    }
    // Element arithmetic on packed FP32 pairs (f32x2: two IEEE round-to-nearest
    // operations per instruction); per-slot constants in registers.
    constexpr int P = V / 2;
    constexpr int SV = V / 4;  // 16-byte FP32 pieces per slot
    f32x2 w[VPT][P], cth[RES ? VPT : 1][P], sth[RES ? VPT : 1][P], nsth[RES ? VPT : 1][P];
    f32x2 acc_g[G ? VPT : 1][P], acc_t[RES ? VPT : 1][P];
    {
        const f32x2 off2 = f2_make(a.gain_offset, a.gain_offset);
        const f32x2 zero = f2_make(0.0f, 0.0f);
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
#pragma unroll
            for (int q = 0; q < P; ++q) {
                w[i][q] = f2_make(1.0f, 1.0f);
                if constexpr (G) {
                    const float2 g2 = __ldg(reinterpret_cast<const float2*>(a.gain + gcol[i]) + q);
                    w[i][q] = f2_add(f2_make(g2.x, g2.y), off2);  // FP32 sums
                    acc_g[i][q] = zero;
                }
                if constexpr (RES) {
                    const float2 t2 = __ldg(reinterpret_cast<const float2*>(a.theta + gcol[i]) + q);
                    float s0, c0, s1, c1;
                    sincosf(t2.x, &s0, &c0);
                    sincosf(t2.y, &s1, &c1);
                    cth[i][q] = f2_make(c0, c1);
                    sth[i][q] = f2_make(s0, s1);
                    nsth[i][q] = f2_make(-s0, -s1);
                    acc_t[i][q] = zero;
                }
            }
        }
    }
    const float inv_width = 1.0f / (float)a.width;
    char* dx_row = static_cast<char*>(a.dx) + r0 * a.dx_stride * (int64_t)sizeof(T);
    const int64_t dx_step = step * a.dx_stride * (int64_t)sizeof(T);
    float* dh_row = RES ? a.dstream_in + r0 * (int64_t)a.width : nullptr;
    const int64_t dh_step = step * (int64_t)a.width;

    bool alive = true;
    int bank = 0;
    int s = 0;
    uint32_t phase = 0;
    for (int k = 0; k < n; ++k) {
        if (alive) alive = mbar_wait(&full_bar[s], phase);
        alive = __all_sync(0xffffffffu, alive);
        const unsigned char* st = smem + s * L.stage_bytes;
        f32x2 x[VPT][P], g[VPT][P], h[RES ? VPT : 1][P];
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const bool rd = alive && valid[i];
            const uint32_t xo = (uint32_t)col[i] * sizeof(T);
            to_pairs<T>(rd ? *reinterpret_cast<const uint4*>(st + xo) : make_uint4(0, 0, 0, 0), x[i]);
            if constexpr (RES) {
#pragma unroll
                for (int q = 0; q < SV; ++q) {
                    const uint32_t fo = (uint32_t)col[i] * 4u + 16u * q;
                    to_pairs<float>(rd ? *reinterpret_cast<const uint4*>(st + L.dy_off + fo) : make_uint4(0, 0, 0, 0),
                                    g[i] + 2 * q);
                    to_pairs<float>(rd ? *reinterpret_cast<const uint4*>(st + L.h_off + fo) : make_uint4(0, 0, 0, 0),
                                    h[i] + 2 * q);
                }
            } else {
                to_pairs<T>(rd ? *reinterpret_cast<const uint4*>(st + L.dy_off + xo) : make_uint4(0, 0, 0, 0), g[i]);
            }
        }
        // this warp is done with the stage
        __syncwarp();
        if (lane == 0 && alive) mbar_arrive(&empty_bar[s]);
        if (++s == S) {
            s = 0;
            phase ^= 1u;
        }

        // core 5: the blend's gradient reaching the cast branch, rounded to it
        f32x2 dh[RES ? VPT : 1][P];
        if constexpr (RES) {
#pragma unroll
            for (int i = 0; i < VPT; ++i)
#pragma unroll
                for (int q = 0; q < P; ++q) {
                    dh[i][q] = g[i][q];
                    g[i][q] = round_pair<T>(f2_mul(sth[i][q], dh[i][q]));
                }
        }
        // row sums: mean square of the normalised input, gradient dot product
        f32x2 ss2 = f2_make(0.0f, 0.0f), cd2 = f2_make(0.0f, 0.0f);
#pragma unroll
        for (int i = 0; i < VPT; ++i)
#pragma unroll
            for (int q = 0; q < P; ++q) {
                const f32x2 u = FIRST ? f2_mul(x[i][q], w[i][q]) : x[i][q];
                ss2 = f2_fma(u, u, ss2);
                cd2 = f2_fma(FIRST ? g[i][q] : f2_mul(g[i][q], w[i][q]), u, cd2);
            }
        float2 tot = consumer_sum2(f2_sum(ss2), f2_sum(cd2), red, bank, ncons);
        if constexpr (CL > 1) {
            // send this part's sums to every peer (lane p of warp 0 to rank p)
            const int j = k & 1;
            if (tid < CL && (uint32_t)tid != crank)
                push_to_peer(peer_addr(&xval[j][crank][0], (uint32_t)tid), peer_addr(&xbar[j], (uint32_t)tid), tot.x,
                             tot.y);
            if (alive) alive = mbar_wait_cluster(&xbar[j], (uint32_t)((k >> 1) & 1));
            alive = __all_sync(0xffffffffu, alive);
            // the parts' sums added in rank order (the same bits in every CTA)
            float sx = 0.0f, sy = 0.0f;
#pragma unroll
            for (int p = 0; p < CL; ++p) {
                const float px = (uint32_t)p == crank ? tot.x : xval[j][p][0];
                const float py = (uint32_t)p == crank ? tot.y : xval[j][p][1];
                sx = p == 0 ? px : sx + px;
                sy = p == 0 ? py : sy + py;
            }
            // the slot's next use is row k + 2, which a peer sends only after
            // this CTA's row k + 1 sums, i.e. after every consumer read it above
            if (tid == 0 && alive && k + 2 < n) mbar_arrive_expect_tx(&xbar[j], kXBytes);
            tot = make_float2(sx, sy);
        }
        const float r = inv_rms_fast(tot.x, inv_width, a.eps);
        const float cr = r * r * r * tot.y * inv_width;
        const f32x2 r2 = f2_make(r, r), ncr2 = f2_make(-cr, -cr);

#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            f32x2 d[P];
#pragma unroll
            for (int q = 0; q < P; ++q) {
                if constexpr (FIRST) {
                    // dz = r g - cr x w as x (-cr w) + r g: the first pass's x w
                    // then dies at the barrier instead of staying live across it
                    // (that held 16 more registers; at 8192 columns it spilled)
                    const f32x2 dz = f2_fma(x[i][q], f2_mul(ncr2, w[i][q]), f2_mul(r2, g[i][q]));
                    d[q] = f2_mul(dz, w[i][q]);
                    if constexpr (G) acc_g[i][q] = f2_fma(dz, x[i][q], acc_g[i][q]);
                } else {
                    d[q] = f2_fma(x[i][q], ncr2, f2_mul(f2_mul(r2, w[i][q]), g[i][q]));
                    if constexpr (G) acc_g[i][q] = f2_fma(g[i][q], f2_mul(x[i][q], r2), acc_g[i][q]);
                }
            }
            if (alive && valid[i]) st_vec(dx_row + (uint32_t)gcol[i] * sizeof(T), from_pairs<T>(d));
            if constexpr (RES) {
                f32x2 dhs[P];
#pragma unroll
                for (int q = 0; q < P; ++q) {
                    dhs[q] = f2_mul(cth[i][q], dh[i][q]);
                    const f32x2 v = FIRST ? f2_mul(f2_mul(x[i][q], w[i][q]), r2) : f2_mul(f2_mul(x[i][q], r2), w[i][q]);
                    const f32x2 nb = round_pair<T>(v);  // the forward's cast branch
                    acc_t[i][q] = f2_fma(dh[i][q], f2_fma(nsth[i][q], h[i][q], f2_mul(cth[i][q], nb)), acc_t[i][q]);
                }
                if (alive && valid[i]) {
#pragma unroll
                    for (int q = 0; q < SV; ++q)
                        st_vec(dh_row + gcol[i] + 4 * q, from_pairs<float>(dhs + 2 * q));
                }
            }
        }
        dx_row += dx_step;
        if constexpr (RES) dh_row += dh_step;
    }

    // one partial row of the parameter gradients per CTA
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        if (!valid[i]) continue;
        if constexpr (G)
            if (a.part_gain)
#pragma unroll
                for (int q = 0; q < SV; ++q)
                    st_vec(a.part_gain + r0 * a.width + gcol[i] + 4 * q, from_pairs<float>(acc_g[i] + 2 * q));
        if constexpr (RES)
            if (a.part_theta)
#pragma unroll
                for (int q = 0; q < SV; ++q)
                    st_vec(a.part_theta + r0 * a.width + gcol[i] + 4 * q, from_pairs<float>(acc_t[i] + 2 * q));
    }
    // no CTA of a cluster exits while a peer may still write to it
    if constexpr (CL > 1) cluster_sync_all();
}

// One entry symbol per core.
template <typename T, int VPT, bool G, int S, int CL>
__global__ void __launch_bounds__(VPT == 1 ? 544 : 288, VPT == 2 ? 2 : 1) rms_norm_bwd_kernel(const __grid_constant__ RowBwdArgs a) {
    pdl_begin();
    row_bwd_body<T, BwdOp::kRms, VPT, G, S, CL>(a);
}
template <typename T, int VPT, bool G, int S, int CL>
__global__ void __launch_bounds__(VPT == 1 ? 544 : 288, VPT == 2 ? 2 : 1) input_scale_norm_bwd_kernel(const __grid_constant__ RowBwdArgs a) {
    pdl_begin();
    row_bwd_body<T, BwdOp::kInputScale, VPT, G, S, CL>(a);
}
template <typename T, int VPT, bool G, int S, int CL>
__global__ void __launch_bounds__(512 + 32) norm_residual_bwd_kernel(const __grid_constant__ RowBwdArgs a) {
    pdl_begin();
    row_bwd_body<T, BwdOp::kResidual, VPT, G, S, CL>(a);
}
template <typename T, int VPT, bool G, int S, int CL>
__global__ void __launch_bounds__(512 + 32) norm_residual_input_scale_bwd_kernel(const __grid_constant__ RowBwdArgs a) {
    pdl_begin();
    row_bwd_body<T, BwdOp::kResidualIS, VPT, G, S, CL>(a);
}

template <typename T, BwdOp OP, int VPT, bool G, int S, int CL>
constexpr auto row_bwd_kernel() {
    if constexpr (OP == BwdOp::kRms) return rms_norm_bwd_kernel<T, VPT, G, S, CL>;
    else if constexpr (OP == BwdOp::kInputScale) return input_scale_norm_bwd_kernel<T, VPT, G, S, CL>;
    else if constexpr (OP == BwdOp::kResidual) return norm_residual_bwd_kernel<T, VPT, G, S, CL>;
    else return norm_residual_input_scale_bwd_kernel<T, VPT, G, S, CL>;
}

// out[c] = sum over parts of part[p][c], in a fixed order: 32 thread groups
// each sum the parts p = grp (mod 32) in order, then one warp adds the 32
// results in a fixed tree (many short runs keep many loads in flight).
constexpr int kReduceGroups = 32;
__global__ void __launch_bounds__(32 * kReduceGroups) param_grad_reduce_kernel(const float* __restrict__ part,
                                                                               int nparts, int width,
                                                                               float* __restrict__ out) {
    pdl_begin();
    __shared__ float sm[kReduceGroups][33];
    const int lane = threadIdx.x & 31, grp = threadIdx.x >> 5;
    const int c = blockIdx.x * 32 + lane;
    float acc = 0.0f;
    if (c < width)
        for (int p = grp; p < nparts; p += kReduceGroups) acc += part[(int64_t)p * width + c];
    sm[grp][lane] = acc;
    __syncthreads();
    if (grp == 0) {
        float v[kReduceGroups];
#pragma unroll
        for (int q = 0; q < kReduceGroups; ++q) v[q] = sm[q][lane];
#pragma unroll
        for (int n = kReduceGroups / 2; n > 0; n >>= 1)
#pragma unroll
            for (int q = 0; q < n; ++q) v[q] += v[q + n];
        if (c < width) out[c] = v[0];
    }
}

int bwd_grid_cap() { return kBwdMaxCtasPerSm * sm_count(); }

// Clusters of `cl` CTAs of `kernel` that can be resident at once (cached).
int resident_clusters(const void* kernel, int threads, size_t smem, int cl) {
    static std::mutex mu;
    static std::map<std::tuple<const void*, int, int, size_t>, int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 1;
    const auto key = std::make_tuple(kernel, threads, dev, smem);
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cl * (unsigned)sm_count());
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n < 1) {
        (void)cudaGetLastError();
        n = 1;
    }
    cache[key] = n;
    return n;
}

// Launch in clusters of `cl` CTAs along x (stream-ordered: no programmatic
// dependent launch, which slowed four-CTA clusters launched back to back).
template <typename... KArgs, typename... Args>
cudaError_t launch_cluster(void (*kernel)(KArgs...), unsigned cl, unsigned grid, unsigned block, size_t smem,
                           cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Launch shape of one instance: threads, dynamic shared memory and the grid
// (resident CTAs x SMs, at most kBwdMaxCtasPerSm per SM and one CTA per row).
// With plan_only the kernel is not launched (the grid is what a launch of the
// same arguments on the current device would use).
// CL > 1: clusters of CL CTAs split each row (the grid counts CTAs; one
// partial row of the parameter gradients per cluster).
template <typename T, BwdOp OP, int VPT, bool G, int S, int CL = 1>
cudaError_t launch_bwd_s(RowBwdArgs a, int nvec, float* dgain, float* dtheta, cudaStream_t s,
                         int64_t* plan_grid = nullptr) {
    const int ncons = ((nvec / CL + VPT - 1) / VPT + 31) / 32 * 32;
    const int threads = ncons + 32;
    const BwdLayout L = bwd_layout<T, OP>(a.width / CL);
    const size_t smem = (size_t)S * L.stage_bytes;
    auto kern = row_bwd_kernel<T, OP, VPT, G, S, CL>();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int64_t units;  // CTAs (CL = 1) or clusters (CL > 1): one per row at most
    if constexpr (CL == 1) {
        const int per_sm = min(blocks_per_sm((const void*)kern, threads, smem), kBwdMaxCtasPerSm);
        units = (int64_t)per_sm * sm_count();
    } else {
        units = min((int64_t)resident_clusters((const void*)kern, threads, smem, CL), (int64_t)bwd_grid_cap() / CL);
    }
    if (units > a.rows) units = a.rows;
    if (units < 1) units = 1;
    const int64_t grid = units * CL;
    if (plan_grid) {
        *plan_grid = units;
        return cudaSuccess;
    }
    if (!(G && dgain)) a.part_gain = nullptr;
    if (!dtheta) a.part_theta = nullptr;
    if constexpr (CL == 1)
        e = launch_pdl(kern, (unsigned)grid, (unsigned)threads, smem, s, a);
    else
        e = launch_cluster(kern, (unsigned)CL, (unsigned)grid, (unsigned)threads, smem, s, a);
    if (e != cudaSuccess) return e;
    const unsigned rgrid = (unsigned)((a.width + 31) / 32);
    if (a.part_gain) {
        e = launch_pdl(param_grad_reduce_kernel, rgrid, 32u * kReduceGroups, 0, s, (const float*)a.part_gain, (int)units, (int)a.width, dgain);
        if (e != cudaSuccess) return e;
    }
    if constexpr (b_is_res(OP)) {
        if (a.part_theta)
            e = launch_pdl(param_grad_reduce_kernel, rgrid, 32u * kReduceGroups, 0, s, (const float*)a.part_theta, (int)units, (int)a.width, dtheta);
    }
    return e;
}

template <typename T, BwdOp OP, int VPT, int CL = 1>
cudaError_t launch_bwd_v(const RowBwdArgs& a, int nvec, float* dgain, float* dtheta, cudaStream_t s,
                         int64_t* plan_grid) {
    const BwdLayout L = bwd_layout<T, OP>(a.width / CL);
    const bool g = a.gain != nullptr;
    // three stages up to 16 KB (cores 1, 2 at 4096 bf16 columns: 3% faster
    // than two); core 5's 40 KB stages stay at two (three measured slower)
    if (L.stage_bytes <= 16 * 1024)
        return g ? launch_bwd_s<T, OP, VPT, true, 3, CL>(a, nvec, dgain, dtheta, s, plan_grid)
                 : launch_bwd_s<T, OP, VPT, false, 3, CL>(a, nvec, dgain, dtheta, s, plan_grid);
    return g ? launch_bwd_s<T, OP, VPT, true, 2, CL>(a, nvec, dgain, dtheta, s, plan_grid)
             : launch_bwd_s<T, OP, VPT, false, 2, CL>(a, nvec, dgain, dtheta, s, plan_grid);
}

// Slots per consumer thread: one up to 256 vectors (core 5: 512), then two,
// then four (cores 1, 2).  Core 5 rows of more than 512 vectors (up to 1024)
// go to a cluster of kSplitCtas CTAs (or two when the count does not divide
// by it) with one slot per thread each.
template <typename T, BwdOp OP>
cudaError_t launch_bwd_op(const RowBwdArgs& a, float* dgain, float* dtheta, cudaStream_t s,
                          int64_t* plan_grid) {
    const int nvec = a.width / Vec<T>::N;
    if (nvec <= 256 || (b_is_res(OP) && nvec <= 512))
        return launch_bwd_v<T, OP, 1>(a, nvec, dgain, dtheta, s, plan_grid);
    if constexpr (b_is_res(OP)) {
        if constexpr (kSplitCtas == 4)
            if (nvec % 4 == 0 && nvec <= 1024) return launch_bwd_v<T, OP, 1, 4>(a, nvec, dgain, dtheta, s, plan_grid);
        if (nvec % 2 == 0 && nvec <= 1024) return launch_bwd_v<T, OP, 1, 2>(a, nvec, dgain, dtheta, s, plan_grid);
        return launch_bwd_v<T, OP, 2>(a, nvec, dgain, dtheta, s, plan_grid);
    } else {
        if (nvec <= 512) return launch_bwd_v<T, OP, 2>(a, nvec, dgain, dtheta, s, plan_grid);
        return launch_bwd_v<T, OP, 4>(a, nvec, dgain, dtheta, s, plan_grid);
    }
}

template <typename T>
cudaError_t launch_bwd_t(BwdOp op, const RowBwdArgs& a, float* dgain, float* dtheta, cudaStream_t s,
                         int64_t* plan_grid = nullptr) {
    switch (op) {
        case BwdOp::kRms: return launch_bwd_op<T, BwdOp::kRms>(a, dgain, dtheta, s, plan_grid);
        case BwdOp::kInputScale: return launch_bwd_op<T, BwdOp::kInputScale>(a, dgain, dtheta, s, plan_grid);
        case BwdOp::kResidual: return launch_bwd_op<T, BwdOp::kResidual>(a, dgain, dtheta, s, plan_grid);
        case BwdOp::kResidualIS: return launch_bwd_op<T, BwdOp::kResidualIS>(a, dgain, dtheta, s, plan_grid);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

// Fixed scratch of the allocation-free gain-gradient call: one partial row
// per CTA of the core 1 backward, kNoAllocScratchBytes at most (16 MiB: 1024
// partial rows of 4096 FP32 columns).
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

cudaError_t noalloc_scratch(void** ptr) {
    static std::mutex mu;
    static std::map<int, void*> addr;  // per device, taken once
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    auto it = addr.find(dev);
    if (it == addr.end()) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        it = addr.emplace(dev, p).first;
    }
    *ptr = it->second;
    return cudaSuccess;
}

size_t row_bwd_gain_scratch_bytes(int64_t rows, int32_t width) {
    const int64_t grid = min(rows, (int64_t)bwd_grid_cap());
    return (size_t)(grid < 1 ? 1 : grid) * (size_t)width * sizeof(float);
}

cudaError_t row_bwd_launch_grid(int dtype, BwdOp op, const RowBwdArgs& a, int64_t* grid) {
    return dtype == 0 ? launch_bwd_t<__nv_bfloat16>(op, a, nullptr, nullptr, nullptr, grid)
                      : launch_bwd_t<float>(op, a, nullptr, nullptr, nullptr, grid);
}

size_t row_bwd_workspace_bytes(int64_t rows, int32_t width) {
    const int64_t grid = min(rows, (int64_t)bwd_grid_cap());
    return (size_t)(grid < 1 ? 1 : grid) * (size_t)width * sizeof(float) * 2;
}

cudaError_t launch_param_grad_reduce(const float* part, int nparts, int width, float* out, cudaStream_t s) {
    const unsigned rgrid = (unsigned)((width + 31) / 32);
    return launch_pdl(param_grad_reduce_kernel, rgrid, 32u * kReduceGroups, 0, s, part, nparts, width, out);
}

cudaError_t launch_row_bwd(int dtype, BwdOp op, RowBwdArgs a, float* dgain, float* dtheta, cudaStream_t s) {
    return dtype == 0 ? launch_bwd_t<__nv_bfloat16>(op, a, dgain, dtheta, s)
                      : launch_bwd_t<float>(op, a, dgain, dtheta, s);
}

cudaError_t read_bwd_device_error(unsigned int* out, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_device_error, sizeof(unsigned int));
    if (e == cudaSuccess && clear) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned int));
    }
    return e;
}

}  // namespace muse
