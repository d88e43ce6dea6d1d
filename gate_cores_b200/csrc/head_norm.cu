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
__device__ unsigned int g_device_error;  // nonzero: an mbarrier wait of the Q/K ring timed out
}  // namespace
}  // namespace muse

#include "tma_pipe.cuh"

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
// one of `split` ranges of that token's head steps).  The token's query heads
// and then its key heads are walked in steps of RW heads (L lanes x one
// 16-byte vector per head); the steps are grouped in batches of BATCH, and
// each warp streams its batches through its own ring of R shared-memory slots
// with cp.async.bulk (one request per batch, issued by lane 0, completed on
// the slot's mbarrier).  The first R batches go out before anything else, so
// the CTA builds its cos/sin table - one sincosf per pair per token, shared by
// all heads of the token - while they are in flight; a slot is refilled as
// soon as the warp has read it, so every warp keeps R batches in flight
// without holding them in registers.  Element arithmetic runs on packed FP32
// pairs in the rotation-pair packing of to_eo (two packed multiply-adds per
// two rotations).  TAIL = false is the instance for shapes without partial
// vectors, heads or batches (every predicate drops out).  Every mbarrier wait
// is bounded; a timeout sets the error word and the warp stops, after its
// copies in flight have landed (bounded again).
template <typename T, int L, bool ROPE, bool UPCAST, bool TAIL, int BATCH, int R, int MINB>
__global__ void __launch_bounds__(256, MINB) qk_norm_rope_kernel(const __grid_constant__ QkArgs a) {
    pdl_begin();
    constexpr int V = Vec<T>::N;
    constexpr int H = qk::EoPack<T>::H;
    constexpr int RW = 32 / L;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t bars[8][R];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    const int split = a.split;
    const int tt = nwarps / split;
    const int sub = lane % L;
    const int slot = lane / L;
    const int nvec = a.head_dim / V;
    const int half = a.head_dim / 2;
    const float inv_width = 1.0f / (float)a.head_dim;
    const int64_t t0 = (int64_t)blockIdx.x * tt;
    const int ntok = (int)min((int64_t)tt, a.tokens - t0);
    float* cs = reinterpret_cast<float*>(smem_raw);
    float* sn = cs + tt * half;
    const int tok = warp / split;
    const int part = warp - tok * split;
    const int64_t t = t0 + tok;
    const uint32_t head_bytes = (uint32_t)a.head_dim * sizeof(T);
    const uint32_t slot_bytes = (BATCH * RW * head_bytes + 127u) & ~127u;
    unsigned char* ring = smem_raw + ((2u * tt * half * 4u + 127u) & ~127u) + (uint32_t)warp * R * slot_bytes;

    const int nst_q = (a.hq + RW - 1) / RW;
    const int nst = nst_q + (a.hkv + RW - 1) / RW;
    const int spw = (nst + split - 1) / split;
    const int g_begin = part * spw, g_end = min(nst, g_begin + spw);
    const int q_hi = min(g_end, nst_q);
    const int k_lo = max(g_begin, nst_q) - nst_q, k_hi = g_end - nst_q;
    const int nbq = q_hi > g_begin ? (q_hi - g_begin + BATCH - 1) / BATCH : 0;
    const int nbk = k_hi > k_lo ? (k_hi - k_lo + BATCH - 1) / BATCH : 0;
    const int nb = tok < ntok ? nbq + nbk : 0;
    const char* q_src = static_cast<const char*>(a.q) + t * a.q_stride * (int64_t)sizeof(T);
    const char* k_src = static_cast<const char*>(a.k) + t * a.k_stride * (int64_t)sizeof(T);

    // batch j: first step, end of its segment, head count, source row
    auto batch = [&](int j, int& st0, int& s_hi, int& count, bool& isq) {
        isq = j < nbq;
        st0 = isq ? g_begin + j * BATCH : k_lo + (j - nbq) * BATCH;
        s_hi = isq ? q_hi : k_hi;
        count = isq ? a.hq : a.hkv;
    };
    auto issue = [&](int j) {
        int st0, s_hi, count;
        bool isq;
        batch(j, st0, s_hi, count, isq);
        const int h0 = st0 * RW, h1 = min(count, min(st0 + BATCH, s_hi) * RW);
        const uint32_t bytes = (uint32_t)(h1 - h0) * head_bytes;
        uint64_t* bar = &bars[warp][j % R];
        pipe::mbar_arrive_expect_tx(bar, bytes);
        pipe::bulk_g2s(ring + (j % R) * slot_bytes, (isq ? q_src : k_src) + (uint32_t)h0 * head_bytes, bytes, bar);
    };
    int issued = 0;
    if (lane == 0 && nb > 0) {
        for (int r = 0; r < R; ++r) pipe::mbar_init(&bars[warp][r], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (; issued < min(R, nb); ++issued) issue(issued);
    }
    __syncwarp();

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
    if (nb == 0) return;

    const bool vok = !TAIL || sub < nvec;
    const uint32_t voff = (uint32_t)sub * 16u;
    // v2 rotation with bf16 Q/K: the rotation on bf16 pairs (qk::bf2_mul /
    // bf2_add give the bf16 products and their rounded sums)
    constexpr bool BF2 = ROPE && !UPCAST && std::is_same<T, __nv_bfloat16>::value;
    f32x2 c2[H], s2[H], n2[H];
    uint32_t cb[BF2 ? H : 1], sb[BF2 ? H : 1], nb2[BF2 ? H : 1];
    if constexpr (ROPE) {
        const int tb = tok * half + (vok ? sub * (V / 2) : 0);
#pragma unroll
        for (int j = 0; j < H; ++j) {
            c2[j] = *reinterpret_cast<const f32x2*>(cs + tb + 2 * j);
            s2[j] = *reinterpret_cast<const f32x2*>(sn + tb + 2 * j);
            n2[j] = f2_mul(s2[j], f2_make(-1.0f, -1.0f));
            if constexpr (BF2) {  // exact: the table holds bf16 values
                float lo, hi;
                f2_split(c2[j], lo, hi);
                cb[j] = pack_bf16x2(lo, hi);
                f2_split(s2[j], lo, hi);
                sb[j] = pack_bf16x2(lo, hi);
                nb2[j] = pack_bf16x2(-lo, -hi);
            }
        }
    }
    const f32x2 qs2 = f2_make(a.query_scale, a.query_scale);
    const bool scaled = a.query_scale != 1.0f;
    char* q_dst = static_cast<char*>(a.q_out) + t * a.q_out_stride * (int64_t)sizeof(T) + (uint32_t)slot * head_bytes;
    char* k_dst = static_cast<char*>(a.k_out) + t * a.k_out_stride * (int64_t)sizeof(T) + (uint32_t)slot * head_bytes;

    auto compute = [&](auto scale_tag, const uint4 (&xv)[BATCH], const bool (&hv)[BATCH], char* dst) {
        constexpr bool SCALE = decltype(scale_tag)::value;
#pragma unroll
        for (int b = 0; b < BATCH; ++b) {
            f32x2 e[H], o[H];
            f32x2 acc = f2_make(0.0f, 0.0f);
            qk::to_eo<T>(xv[b], e, o);
#pragma unroll
            for (int j = 0; j < H; ++j) {
                acc = f2_fma(e[j], e[j], acc);
                acc = f2_fma(o[j], o[j], acc);
            }
            const float r = inv_rms_fast(group_sum<L>(f2_sum(acc)), inv_width, a.eps);
            const f32x2 r2 = f2_make(r, r);
            if constexpr (BF2) {
                static_assert(H == 2, "a 16-byte vector holds 4 rotation pairs of bf16");
                uint32_t w[4];
#pragma unroll
                for (int j = 0; j < H; ++j) {
                    f32x2 ev = f2_mul(e[j], r2), ov = f2_mul(o[j], r2);
                    if constexpr (SCALE) {  // cast, query_scale, cast again (the last cast below)
                        ev = f2_mul(round_pair<T>(ev), qs2);
                        ov = f2_mul(round_pair<T>(ov), qs2);
                    }
                    float lo, hi;
                    f2_split(ev, lo, hi);
                    const uint32_t eb = pack_bf16x2(lo, hi);  // cast to bf16
                    f2_split(ov, lo, hi);
                    const uint32_t ob = pack_bf16x2(lo, hi);
                    const uint32_t er = qk::bf2_add(qk::bf2_mul(eb, cb[j]), qk::bf2_mul(ob, nb2[j]));
                    const uint32_t orr = qk::bf2_add(qk::bf2_mul(eb, sb[j]), qk::bf2_mul(ob, cb[j]));
                    w[2 * j] = qk::lo_halves(er, orr);  // rotation pair 2j: (first, second)
                    w[2 * j + 1] = qk::hi_halves(er, orr);
                }
                if (hv[b]) st_vec(dst + (uint32_t)(b * RW) * head_bytes + voff, make_uint4(w[0], w[1], w[2], w[3]));
            } else {
#pragma unroll
                for (int j = 0; j < H; ++j) {
                    f32x2 ev = round_pair<T>(f2_mul(e[j], r2));  // cast to the Q/K dtype
                    f32x2 ov = round_pair<T>(f2_mul(o[j], r2));
                    if constexpr (SCALE) {                      // query_scale, cast again
                        ev = round_pair<T>(f2_mul(ev, qs2));
                        ov = round_pair<T>(f2_mul(ov, qs2));
                    }
                    if constexpr (ROPE) qk::rope_eo<T, UPCAST>(ev, ov, c2[j], s2[j], n2[j]);
                    e[j] = ev;
                    o[j] = ov;
                }
                if (hv[b]) st_vec(dst + (uint32_t)(b * RW) * head_bytes + voff, qk::from_eo<T>(e, o));
            }
        }
    };

    bool alive = true;
    int j = 0;
#pragma unroll 1
    for (; j < nb; ++j) {
        alive = __all_sync(0xffffffffu, alive && pipe::mbar_wait(&bars[warp][j % R], (uint32_t)((j / R) & 1)));
        if (!alive) break;
        int st0, s_hi, count;
        bool isq;
        batch(j, st0, s_hi, count, isq);
        const unsigned char* sl = ring + (j % R) * slot_bytes + (uint32_t)slot * head_bytes + voff;
        uint4 xv[BATCH];
        bool hv[BATCH];
#pragma unroll
        for (int b = 0; b < BATCH; ++b) {
            hv[b] = vok && (!TAIL || (st0 + b < s_hi && (st0 + b) * RW + slot < count));
            xv[b] = hv[b] ? *reinterpret_cast<const uint4*>(sl + (uint32_t)(b * RW) * head_bytes) : make_uint4(0, 0, 0, 0);
        }
        // the warp is done with the slot: refill it with batch j + R
        __syncwarp();
        if (lane == 0 && issued < nb) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            issue(issued);
            ++issued;
        }
        char* dst = (isq ? q_dst : k_dst) + (uint32_t)(st0 * RW) * head_bytes;
        if (isq && scaled)
            compute(std::true_type{}, xv, hv, dst);
        else
            compute(std::false_type{}, xv, hv, dst);
    }
    // after a timed-out wait: let this warp's copies still in flight land
    if (lane == 0)
        for (int k = j; k < issued; ++k)
            if (!pipe::mbar_wait(&bars[warp][k % R], (uint32_t)((k / R) & 1))) break;
}

constexpr int kThreads = 256;
// Q/K kernel: 4 head steps per batch, a ring of 3 batches per warp (48 KB of
// slots per CTA), registers for 4 resident CTAs (32 warps) per SM.  Measured
// on B200 against persistent grids that balance (token, batch) units over all
// warps: contiguous unit ranges per warp 8% slower at prefill and 20% slower
// at 32k-80k tokens (the warps stream thousands of far-apart windows), units
// dealt round-robin 35% slower (angles and positions recomputed per unit).
// What this one-shot grid loses at prefill is the last wave (8192 tokens on
// 4736 warp slots is 1.73 waves).
constexpr int kQkBatch = 4;
constexpr int kQkRing = 3;
constexpr int kQkMinBlocks = 4;
// Warps (= tokens) per CTA when every warp takes whole tokens.  Seven: four
// CTAs per SM still (64 registers), and 8192 tokens make 1.98 waves of the
// 592 CTA slots instead of 1.73 with eight; measured on B200 at prefill, the
// five-core step 166.6 -> 162.4 us (Q/K alone 29.3 -> 29.0 us back to back),
// 1% faster on the 80k-token packed batch, unchanged at 32k tokens x 8192;
// six, five or four warps per CTA gained nothing.
constexpr int kQkWarpsWhole = 7;

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

template <typename T, int L, bool ROPE, bool UPCAST>
cudaError_t launch_qk_l(const QkArgs& a0, cudaStream_t s) {
    constexpr int RW = 32 / L;
    constexpr int BATCH = kQkBatch;
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
    const int threads = split == 1 ? 32 * kQkWarpsWhole : kThreads;
    const int tt = split == 1 ? kQkWarpsWhole : nwarps / split;
    const uint32_t head_bytes = (uint32_t)a.head_dim * (uint32_t)sizeof(T);
    const size_t table = ((size_t)2 * tt * (a.head_dim / 2) * 4 + 127) & ~(size_t)127;
    const size_t slot = ((size_t)BATCH * RW * head_bytes + 127) & ~(size_t)127;
    const size_t smem = table + (size_t)(threads / 32) * kQkRing * slot;
    const int64_t grid = (a.tokens + tt - 1) / tt;
    const bool exact = split == 1 && a.head_dim / Vec<T>::N == L && a.hq % RW == 0 &&
                       a.hkv % RW == 0 && nst_q % BATCH == 0 && nst_k % BATCH == 0;
    auto kern = exact ? qk_norm_rope_kernel<T, L, ROPE, UPCAST, false, BATCH, kQkRing, kQkMinBlocks>
                      : qk_norm_rope_kernel<T, L, ROPE, UPCAST, true, BATCH, kQkRing, kQkMinBlocks>;
    // the opt-in is needed whenever static + dynamic shared memory passes 48 KB
    // (the mbarriers are static), so it is always set
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, (unsigned)grid, (unsigned)threads, smem, s, a);
}

template <typename T, int L>
cudaError_t launch_qk_modes(int use_rope, int upcast, const QkArgs& a, cudaStream_t s) {
    if (!use_rope) return launch_qk_l<T, L, false, true>(a, s);
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        if (!upcast) return launch_qk_l<T, L, true, false>(a, s);
    }
    return launch_qk_l<T, L, true, true>(a, s);
}

// Lanes per head: the head's 16-byte vectors rounded up to a power of two
// (heads are at most 512 bytes, so one vector per lane always suffices).
template <typename T>
cudaError_t launch_qk_t(int use_rope, int upcast, const QkArgs& a, cudaStream_t s) {
    const int nv = a.head_dim / Vec<T>::N;
    if (nv > 16) return launch_qk_modes<T, 32>(use_rope, upcast, a, s);
    if (nv <= 1) return launch_qk_modes<T, 1>(use_rope, upcast, a, s);
    if (nv <= 2) return launch_qk_modes<T, 2>(use_rope, upcast, a, s);
    if (nv <= 4) return launch_qk_modes<T, 4>(use_rope, upcast, a, s);
    if (nv <= 8) return launch_qk_modes<T, 8>(use_rope, upcast, a, s);
    return launch_qk_modes<T, 16>(use_rope, upcast, a, s);
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

cudaError_t read_qk_device_error(unsigned int* out, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_device_error, sizeof(unsigned int));
    if (e == cudaSuccess && clear) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned int));
    }
    return e;
}

}  // namespace muse
