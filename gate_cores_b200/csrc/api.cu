// C ABI of the normalisation cores: argument validation, aliasing checks,
// launch configuration and status codes.  Everything here runs on the host;
// no call synchronises or allocates.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <map>
#include <mutex>
#include <initializer_list>
#include <tuple>

#include "kernels.h"
#include "muse_cores.h"

namespace {

thread_local char g_err[512] = "";

muse_status fail(muse_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}

muse_status from_cuda(cudaError_t e, const char* what) {
    if (e == cudaSuccess) return MUSE_OK;
    return fail(MUSE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool valid_dtype(int d) { return d == MUSE_DTYPE_BF16 || d == MUSE_DTYPE_F32; }
int64_t elem_size(int d) { return d == MUSE_DTYPE_BF16 ? 2 : 4; }
int vec_elems(int d) { return d == MUSE_DTYPE_BF16 ? 8 : 4; }
bool aligned(const void* p, uintptr_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }
bool finite(float v) { return std::isfinite(v); }

// Bytes touched by a strided tensor: rows intervals [base + r*stride, + width).
struct Span {
    int64_t base;
    int64_t stride;
    int64_t width;
    int64_t rows;
};

Span span(const void* p, int64_t rows, int64_t width_elems, int64_t stride_elems, int64_t es) {
    return Span{(int64_t)reinterpret_cast<uintptr_t>(p), stride_elems * es, width_elems * es, rows};
}

bool same_span(const Span& a, const Span& b) {
    return a.base == b.base && a.stride == b.stride && a.width == b.width && a.rows == b.rows;
}

int64_t floor_div(int64_t a, int64_t b) {  // b > 0
    int64_t q = a / b;
    if ((a % b != 0) && (a < 0)) --q;
    return q;
}

// True when any byte of a lies in b.  Exact for equal strides (or a single
// row on either side); conservative (bounding ranges) otherwise.
bool overlap(Span a, Span b) {
    if (a.rows <= 0 || b.rows <= 0 || a.width <= 0 || b.width <= 0) return false;
    const int64_t a_end = a.base + (a.rows - 1) * a.stride + a.width;
    const int64_t b_end = b.base + (b.rows - 1) * b.stride + b.width;
    if (a_end <= b.base || b_end <= a.base) return false;
    if (a.rows == 1) a.stride = b.stride;
    if (b.rows == 1) b.stride = a.stride;
    if (a.stride != b.stride || a.stride <= 0) return true;
    // Rows ra of a and rb of b meet iff, with k = rb - ra and d = b.base - a.base,
    // -b.width < d + k * stride < a.width.
    const int64_t S = a.stride, d = b.base - a.base;
    int64_t kmin = floor_div(-b.width - d, S) + 1;
    int64_t kmax = -floor_div(-(a.width - d), S) - 1;  // ceil((a.width - d) / S) - 1
    if (kmin < -(a.rows - 1)) kmin = -(a.rows - 1);
    if (kmax > b.rows - 1) kmax = b.rows - 1;
    return kmin <= kmax;
}

// An output may coincide exactly with one input; any other overlap with any
// tensor of the call is an error.
bool bad_alias(const Span& out, const Span& other, bool may_coincide) {
    if (may_coincide && same_span(out, other)) return false;
    return overlap(out, other);
}

// probe: the bounded-wait probe of muse_rms_norm_stall_probe (spin_limit
// polls per wait; the stage of row stall_row is never signalled).
muse_status row_entry(muse::RowOp op, const void* x, void* y, muse_dtype dtype, int64_t rows,
                      int64_t hidden, int64_t xs, int64_t ys, const float* gain,
                      float gain_offset, float eps, cudaStream_t stream, const char* name,
                      bool probe = false, uint32_t spin_limit = 0, int64_t stall_row = 0) {
    if (!valid_dtype(dtype)) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: unknown dtype %d", name, (int)dtype);
    if (rows < 0 || hidden <= 0)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: rows=%lld hidden=%lld", name, (long long)rows, (long long)hidden);
    if (!finite(eps) || eps < 0.0f || !finite(gain_offset))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: eps must be finite and >= 0, gain_offset finite", name);
    if (xs < hidden || ys < hidden)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: row strides must be >= hidden", name);
    if (rows == 0) return MUSE_OK;
    if (!x || !y) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: null x or y", name);
    const int64_t es = elem_size(dtype);
    if (!aligned(x, 16) || !aligned(y, 16) || (hidden * es) % 16 || (xs * es) % 16 || (ys * es) % 16)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: pointers, row widths and strides must be 16-byte multiples", name);
    if (gain && !aligned(gain, 16)) return fail(MUSE_ERR_UNSUPPORTED, "%s: gain not 16-byte aligned", name);
    if (hidden * es > MUSE_MAX_ROW_BYTES)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: row of %lld bytes exceeds %d", name, (long long)(hidden * es), MUSE_MAX_ROW_BYTES);
    if (probe) {
        // the probe needs the bulk-copy pipeline, which rows up to 1024 16-byte vectors take
        if (hidden * es > 16384)
            return fail(MUSE_ERR_UNSUPPORTED, "%s: probe rows are limited to 16384 bytes", name);
        if (spin_limit < 1 || spin_limit > (1u << 24) || stall_row < 0 || stall_row >= rows)
            return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: spin_limit in [1, 2^24] and stall_row in [0, rows) required",
                        name);
    }
    const Span sx = span(x, rows, hidden, xs, es), sy = span(y, rows, hidden, ys, es);
    if (bad_alias(sy, sx, true) || (gain && bad_alias(sy, span(gain, 1, hidden, hidden, 4), false)))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: output partially overlaps an input", name);
    muse::RowArgs a{};
    a.x = x;
    a.y = y;
    a.gain = gain;
    a.rows = rows;
    a.x_stride = xs;
    a.y_stride = ys;
    a.width = (int32_t)hidden;
    a.gain_offset = gain_offset;
    a.eps = eps;
    if (probe) {
        a.spin_limit = spin_limit;
        a.probe_stall = 1;
        a.stall_row = stall_row;
    }
    return from_cuda(muse::launch_row(dtype, op, a, stream), name);
}

// Shared checks of the row backward entry points: the workspace and the
// parameter-gradient outputs must not overlap each other or any tensor.
muse_status bwd_workspace_check(const char* name, size_t need, void* ws, size_t ws_bytes,
                                bool needed) {
    if (!needed) return MUSE_OK;
    if (!ws || ws_bytes < need)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: workspace of %zu bytes needed, %zu given", name, need,
                    ws ? ws_bytes : (size_t)0);
    if (!aligned(ws, 16)) return fail(MUSE_ERR_UNSUPPORTED, "%s: workspace not 16-byte aligned", name);
    return MUSE_OK;
}

bool any_overlap(const Span& a, std::initializer_list<Span> others) {
    for (const Span& o : others)
        if (overlap(a, o)) return true;
    return false;
}

// noalloc: the gain partials go to the library's fixed device array instead
// of the caller's workspace (ws / ws_bytes ignored); its size is checked
// against the grid this launch will use, and its address is looked up only
// after every argument check has passed.
muse_status row_bwd_entry(bool input_scale, const void* x, const void* dy, void* dx,
                          muse_dtype dtype, int64_t rows, int64_t hidden, int64_t xs,
                          int64_t dys, int64_t dxs, const float* gain, float gain_offset,
                          float eps, float* dgain, void* ws, size_t ws_bytes, cudaStream_t stream,
                          const char* name, bool noalloc = false) {
    if (!valid_dtype(dtype)) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: unknown dtype %d", name, (int)dtype);
    if (rows < 0 || hidden <= 0)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: rows=%lld hidden=%lld", name, (long long)rows, (long long)hidden);
    if (!finite(eps) || eps < 0.0f || !finite(gain_offset))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: eps must be finite and >= 0, gain_offset finite", name);
    if (xs < hidden || dys < hidden || dxs < hidden)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: row strides must be >= hidden", name);
    if (dgain && !gain) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: dgain requested without a gain", name);
    if (rows == 0) {
        if (dgain) return from_cuda(cudaMemsetAsync(dgain, 0, sizeof(float) * (size_t)hidden, stream), name);
        return MUSE_OK;
    }
    if (!x || !dy || !dx) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: null x, dy or dx", name);
    const int64_t es = elem_size(dtype);
    if (!aligned(x, 16) || !aligned(dy, 16) || !aligned(dx, 16) || (hidden * es) % 16 || (xs * es) % 16 ||
        (dys * es) % 16 || (dxs * es) % 16)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: pointers, row widths and strides must be 16-byte multiples", name);
    if ((gain && !aligned(gain, 16)) || (dgain && !aligned(dgain, 16)))
        return fail(MUSE_ERR_UNSUPPORTED, "%s: gain / dgain not 16-byte aligned", name);
    if (hidden / vec_elems(dtype) > muse::kBwdMaxVectors)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: rows of more than %d 16-byte vectors", name, muse::kBwdMaxVectors);
    const muse::BwdOp op = input_scale ? muse::BwdOp::kInputScale : muse::BwdOp::kRms;
    if (noalloc) ws = nullptr, ws_bytes = 0;
    if (!noalloc) {
        // cores 1 and 2 use the gain half of the workspace only
        muse_status st = bwd_workspace_check(name, muse::row_bwd_gain_scratch_bytes(rows, (int32_t)hidden),
                                             ws, ws_bytes, dgain != nullptr);
        if (st != MUSE_OK) return st;
    }
    const Span sx = span(x, rows, hidden, xs, es), sdy = span(dy, rows, hidden, dys, es);
    const Span sdx = span(dx, rows, hidden, dxs, es);
    const Span sg = span(gain, gain ? 1 : 0, hidden, hidden, 4), sdg = span(dgain, dgain ? 1 : 0, hidden, hidden, 4);
    const Span sws = span(ws, (dgain && ws) ? 1 : 0, (int64_t)ws_bytes, (int64_t)ws_bytes, 1);
    if (bad_alias(sdx, sx, true) || bad_alias(sdx, sdy, true) || any_overlap(sdx, {sg, sdg, sws}) ||
        any_overlap(sdg, {sx, sdy, sg, sws}) || any_overlap(sws, {sx, sdy, sg}))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: an output or the workspace overlaps another tensor", name);
    muse::RowBwdArgs a{};
    a.x = x;
    a.dy = dy;
    a.dx = dx;
    a.gain = gain;
    a.part_gain = static_cast<float*>(ws);
    a.rows = rows;
    a.x_stride = xs;
    a.dy_stride = dys;
    a.dx_stride = dxs;
    a.width = (int32_t)hidden;
    a.gain_offset = gain_offset;
    a.eps = eps;
    if (noalloc && dgain) {
        // the partials of the grid this launch uses: one row of hidden floats per CTA
        int64_t grid = 0;
        muse_status st = from_cuda(muse::row_bwd_launch_grid(dtype, op, a, &grid), name);
        if (st != MUSE_OK) return st;
        const size_t need = (size_t)grid * (size_t)hidden * sizeof(float);
        if (need > muse::kNoAllocScratchBytes)
            return fail(MUSE_ERR_UNSUPPORTED, "%s: gain partials of %lld CTAs need %zu bytes, the fixed scratch holds %zu",
                        name, (long long)grid, need, muse::kNoAllocScratchBytes);
        void* scratch = nullptr;
        st = from_cuda(muse::noalloc_scratch(&scratch), name);
        if (st != MUSE_OK) return st;
        // the library's own array cannot overlap the caller's tensors
        a.part_gain = static_cast<float*>(scratch);
    }
    return from_cuda(muse::launch_row_bwd(dtype, op, a, dgain, nullptr, stream), name);
}

}  // namespace

namespace muse {

int sm_count() {
    static std::mutex mu;
    static std::map<int, int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(dev);
    if (it != cache.end()) return it->second;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev] = n;
    return n;
}

int blocks_per_sm(const void* kernel, int threads, size_t dyn_smem) {
    static std::mutex mu;
    static std::map<std::tuple<const void*, int, int, size_t>, int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 1;
    const auto key = std::make_tuple(kernel, threads, dev, dyn_smem);
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = cache.find(key);
        if (it != cache.end()) return it->second;
    }
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, dyn_smem) != cudaSuccess || n < 1) n = 1;
    std::lock_guard<std::mutex> lock(mu);
    cache[key] = n;
    return n;
}

}  // namespace muse

extern "C" {

int muse_version(void) { return MUSE_VERSION; }

const char* muse_status_string(muse_status s) {
    switch (s) {
        case MUSE_OK: return "MUSE_OK";
        case MUSE_ERR_INVALID_ARGUMENT: return "MUSE_ERR_INVALID_ARGUMENT";
        case MUSE_ERR_UNSUPPORTED: return "MUSE_ERR_UNSUPPORTED";
        case MUSE_ERR_CUDA: return "MUSE_ERR_CUDA";
    }
    return "MUSE_ERR_UNKNOWN";
}

const char* muse_last_error(void) { return g_err; }

muse_status muse_rms_norm(const void* x, void* y, muse_dtype dtype, int64_t rows, int64_t hidden,
                          int64_t x_row_stride, int64_t y_row_stride, const float* gain,
                          float gain_offset, float eps, cudaStream_t stream) {
    return row_entry(muse::RowOp::kRms, x, y, dtype, rows, hidden, x_row_stride, y_row_stride,
                     gain, gain_offset, eps, stream, "muse_rms_norm");
}

muse_status muse_rms_norm_stall_probe(const void* x, void* y, muse_dtype dtype, int64_t rows,
                                      int64_t hidden, int64_t x_row_stride, int64_t y_row_stride,
                                      const float* gain, float gain_offset, float eps,
                                      uint32_t spin_limit, int64_t stall_row, cudaStream_t stream) {
    return row_entry(muse::RowOp::kRms, x, y, dtype, rows, hidden, x_row_stride, y_row_stride,
                     gain, gain_offset, eps, stream, "muse_rms_norm_stall_probe", true, spin_limit,
                     stall_row);
}

muse_status muse_input_scale_norm(const void* x, void* y, muse_dtype dtype, int64_t rows,
                                  int64_t hidden, int64_t x_row_stride, int64_t y_row_stride,
                                  const float* gain, float gain_offset, float eps,
                                  cudaStream_t stream) {
    return row_entry(muse::RowOp::kInputScale, x, y, dtype, rows, hidden, x_row_stride,
                     y_row_stride, gain, gain_offset, eps, stream, "muse_input_scale_norm");
}

muse_status muse_qk_norm_rope(const void* q, const void* k, void* q_out, void* k_out,
                              muse_dtype dtype, muse_layout layout, int64_t batch,
                              int64_t seqlen, const int32_t* cu_seqlens, int32_t num_seqs,
                              int64_t total_tokens, const int32_t* positions, int32_t hq,
                              int32_t hkv, int32_t head_dim, int64_t q_tok_stride,
                              int64_t k_tok_stride, int64_t q_out_tok_stride,
                              int64_t k_out_tok_stride, float eps, float query_scale,
                              int use_rope, int upcast_rope, float rope_base,
                              cudaStream_t stream) {
    const char* name = "muse_qk_norm_rope";
    if (!valid_dtype(dtype)) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: unknown dtype %d", name, (int)dtype);
    if (layout != MUSE_LAYOUT_BSHD && layout != MUSE_LAYOUT_THD)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: unknown layout %d", name, (int)layout);
    int64_t tokens = 0;
    if (layout == MUSE_LAYOUT_BSHD) {
        if (batch < 0 || seqlen < 0 || (batch > 0 && seqlen == 0))
            return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: batch=%lld seqlen=%lld", name, (long long)batch, (long long)seqlen);
        tokens = batch * seqlen;
    } else {
        if (total_tokens < 0 || num_seqs < 0)
            return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: total_tokens=%lld num_seqs=%d", name, (long long)total_tokens, num_seqs);
        tokens = total_tokens;
    }
    if (hq <= 0 || hkv <= 0 || hq % hkv != 0)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: hq=%d must be a positive multiple of hkv=%d", name, hq, hkv);
    if (head_dim <= 0 || (head_dim & 1))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: head_dim=%d must be positive and even", name, head_dim);
    if (!finite(eps) || eps < 0.0f || !finite(query_scale))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: eps must be finite and >= 0, query_scale finite", name);
    if (use_rope && !(finite(rope_base) && rope_base > 0.0f))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: rope_base must be finite and > 0", name);
    const int64_t qw = (int64_t)hq * head_dim, kw = (int64_t)hkv * head_dim;
    if (q_tok_stride < qw || q_out_tok_stride < qw || k_tok_stride < kw || k_out_tok_stride < kw)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: token strides must cover all heads", name);
    const bool derive = use_rope && !positions;
    if (tokens > 0 && derive && layout == MUSE_LAYOUT_THD && (!cu_seqlens || num_seqs < 1))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: THD without positions needs cu_seqlens and num_seqs >= 1", name);
    if (tokens == 0) return MUSE_OK;
    if (!q || !k || !q_out || !k_out) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: null q/k/q_out/k_out", name);
    const int64_t es = elem_size(dtype);
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(q_out, 16) || !aligned(k_out, 16) ||
        (head_dim * es) % 16 || (q_tok_stride * es) % 16 || (k_tok_stride * es) % 16 ||
        (q_out_tok_stride * es) % 16 || (k_out_tok_stride * es) % 16)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: pointers, head_dim and strides must be 16-byte multiples", name);
    if (head_dim / vec_elems(dtype) > 32 || head_dim / 2 > muse::kMaxHalfDim)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: head_dim=%d exceeds 512 bytes per head", name, head_dim);
    if ((positions && !aligned(positions, 4)) || (cu_seqlens && !aligned(cu_seqlens, 4)))
        return fail(MUSE_ERR_UNSUPPORTED, "%s: positions / cu_seqlens not 4-byte aligned", name);
    const Span sq = span(q, tokens, qw, q_tok_stride, es), sk = span(k, tokens, kw, k_tok_stride, es);
    const Span sqo = span(q_out, tokens, qw, q_out_tok_stride, es);
    const Span sko = span(k_out, tokens, kw, k_out_tok_stride, es);
    bool bad = bad_alias(sqo, sq, true) || bad_alias(sqo, sk, false) || bad_alias(sqo, sko, false) ||
               bad_alias(sko, sk, true) || bad_alias(sko, sq, false);
    if (use_rope && positions) {
        const Span sp = span(positions, 1, tokens, tokens, 4);
        bad = bad || bad_alias(sqo, sp, false) || bad_alias(sko, sp, false);
    }
    if (derive && layout == MUSE_LAYOUT_THD) {
        const Span sc = span(cu_seqlens, 1, (int64_t)num_seqs + 1, (int64_t)num_seqs + 1, 4);
        bad = bad || bad_alias(sqo, sc, false) || bad_alias(sko, sc, false);
    }
    if (bad) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: output partially overlaps an input", name);

    muse::QkArgs a{};
    a.q = q;
    a.k = k;
    a.q_out = q_out;
    a.k_out = k_out;
    a.positions = positions;
    a.cu_seqlens = cu_seqlens;
    a.tokens = tokens;
    a.seqlen = layout == MUSE_LAYOUT_BSHD ? seqlen : 1;
    a.q_stride = q_tok_stride;
    a.k_stride = k_tok_stride;
    a.q_out_stride = q_out_tok_stride;
    a.k_out_stride = k_out_tok_stride;
    a.num_seqs = num_seqs;
    a.hq = hq;
    a.hkv = hkv;
    a.head_dim = head_dim;
    a.pos_mode = positions ? 0 : (layout == MUSE_LAYOUT_BSHD ? 1 : 2);
    a.eps = eps;
    a.query_scale = query_scale;
    // FP32 rotary frequencies: base^(-2i/D) evaluated in double, rounded once.
    if (use_rope)
        for (int i = 0; i < head_dim / 2; ++i)
            a.inv_freq[i] = (float)std::pow((double)rope_base, -(2.0 * i) / (double)head_dim);
    return from_cuda(muse::launch_qk(dtype, use_rope, upcast_rope, a, stream), name);
}

muse_status muse_output_norm_gate(const void* o, const void* gate, void* y, muse_dtype dtype,
                                  int64_t tokens, int32_t heads, int32_t head_dim,
                                  int32_t norm_group, float eps, cudaStream_t stream) {
    const char* name = "muse_output_norm_gate";
    if (!valid_dtype(dtype)) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: unknown dtype %d", name, (int)dtype);
    if (tokens < 0 || heads <= 0 || head_dim <= 0)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: tokens=%lld heads=%d head_dim=%d", name, (long long)tokens, heads, head_dim);
    const int64_t width = (int64_t)heads * head_dim;
    if (norm_group != head_dim && norm_group != width)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: norm_group=%d must be head_dim or heads*head_dim", name, norm_group);
    if (!finite(eps) || eps < 0.0f) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: eps must be finite and >= 0", name);
    if (tokens == 0) return MUSE_OK;
    if (!o || !gate || !y) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: null o/gate/y", name);
    const int64_t es = elem_size(dtype);
    if (!aligned(o, 16) || !aligned(gate, 16) || !aligned(y, 16) || (head_dim * es) % 16)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: pointers and head_dim must be 16-byte multiples", name);
    const bool per_head = norm_group == head_dim && head_dim / vec_elems(dtype) <= 32;
    if (!per_head && norm_group * es > MUSE_MAX_ROW_BYTES)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: norm group of %lld bytes exceeds %d", name, (long long)(norm_group * es), MUSE_MAX_ROW_BYTES);
    const Span so = span(o, tokens, width, width, es), sg = span(gate, tokens, width, width, es);
    const Span sy = span(y, tokens, width, width, es);
    if (bad_alias(sy, so, true) || bad_alias(sy, sg, true))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: output partially overlaps an input", name);
    if (per_head) {
        muse::HeadGateArgs a{};
        a.o = o;
        a.gate = gate;
        a.y = y;
        a.rows = tokens * heads;
        a.width = head_dim;
        a.eps = eps;
        return from_cuda(muse::launch_head_gate(dtype, a, stream), name);
    }
    muse::RowArgs a{};
    a.x = o;
    a.gate = gate;
    a.y = y;
    a.rows = tokens * (width / norm_group);
    a.x_stride = a.y_stride = a.gate_stride = norm_group;
    a.width = norm_group;
    a.eps = eps;
    return from_cuda(muse::launch_row(dtype, muse::RowOp::kNormGate, a, stream), name);
}

muse_status muse_norm_residual(const float* stream_in, const void* branch, float* stream_out,
                               muse_dtype branch_dtype, int64_t rows, int64_t hidden,
                               const float* gain, float gain_offset, const float* theta,
                               int input_scale, float norm_eps, cudaStream_t stream) {
    const char* name = "muse_norm_residual";
    if (!valid_dtype(branch_dtype)) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: unknown dtype %d", name, (int)branch_dtype);
    if (rows < 0 || hidden <= 0)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: rows=%lld hidden=%lld", name, (long long)rows, (long long)hidden);
    if (!finite(norm_eps) || norm_eps < 0.0f || !finite(gain_offset))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: norm_eps must be finite and >= 0, gain_offset finite", name);
    if (rows == 0) return MUSE_OK;
    if (!stream_in || !branch || !stream_out || !theta)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: null stream_in/branch/stream_out/theta", name);
    const int64_t es = elem_size(branch_dtype);
    if (!aligned(stream_in, 16) || !aligned(stream_out, 16) || !aligned(branch, 16) || (hidden * es) % 16)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: pointers and row widths must be 16-byte multiples", name);
    if (!aligned(theta, 16) || (gain && !aligned(gain, 16)))
        return fail(MUSE_ERR_UNSUPPORTED, "%s: theta / gain not 16-byte aligned", name);
    if (hidden * es > MUSE_MAX_ROW_BYTES)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: branch row of %lld bytes exceeds %d", name, (long long)(hidden * es), MUSE_MAX_ROW_BYTES);
    const Span sin_ = span(stream_in, rows, hidden, hidden, 4), sout = span(stream_out, rows, hidden, hidden, 4);
    const Span sb = span(branch, rows, hidden, hidden, es), st = span(theta, 1, hidden, hidden, 4);
    bool bad = bad_alias(sout, sin_, true) || bad_alias(sout, sb, false) || bad_alias(sout, st, false);
    if (gain) bad = bad || bad_alias(sout, span(gain, 1, hidden, hidden, 4), false);
    if (bad) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: output partially overlaps an input", name);
    muse::RowArgs a{};
    a.x = branch;
    a.stream_in = stream_in;
    a.stream_out = stream_out;
    a.gain = gain;
    a.theta = theta;
    a.rows = rows;
    a.x_stride = hidden;
    a.s_in_stride = a.s_out_stride = hidden;
    a.width = (int32_t)hidden;
    a.gain_offset = gain_offset;
    a.eps = norm_eps;
    const muse::RowOp op = input_scale ? muse::RowOp::kResidualIS : muse::RowOp::kResidual;
    return from_cuda(muse::launch_row(branch_dtype, op, a, stream), name);
}

}  // extern "C"

namespace {

// Shared checks of the two _residual_core entry points; p is theta or the gate.
muse_status residual_entry(const float* stream_in, const void* branch, float* stream_out,
                           muse_dtype branch_dtype, int64_t rows, int64_t hidden, const float* p,
                           bool gate, float temperature, float eps, cudaStream_t stream, const char* name) {
    if (!valid_dtype(branch_dtype)) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: unknown dtype %d", name, (int)branch_dtype);
    if (rows < 0 || hidden <= 0)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: rows=%lld hidden=%lld", name, (long long)rows, (long long)hidden);
    if (gate && !(finite(temperature) && temperature > 0.0f && finite(eps) && eps >= 0.0f && eps <= 1.0f))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: temperature must be finite and > 0, eps in [0, 1]", name);
    if (rows == 0) return MUSE_OK;
    if (!stream_in || !branch || !stream_out || !p)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: null stream_in/branch/stream_out/%s", name, gate ? "gate" : "theta");
    const int64_t es = elem_size(branch_dtype);
    if (!aligned(stream_in, 16) || !aligned(stream_out, 16) || !aligned(branch, 16) || !aligned(p, 16) ||
        (hidden * es) % 16)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: pointers and row widths must be 16-byte multiples", name);
    if (hidden / vec_elems(branch_dtype) > (int64_t)65535 * 256)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: rows of more than %d 16-byte vectors", name, 65535 * 256);
    const Span sin_ = span(stream_in, rows, hidden, hidden, 4), sout = span(stream_out, rows, hidden, hidden, 4);
    const Span sb = span(branch, rows, hidden, hidden, es), sp = span(p, 1, hidden, hidden, 4);
    if (bad_alias(sout, sin_, true) || bad_alias(sout, sb, false) || bad_alias(sout, sp, false))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: output partially overlaps an input", name);
    muse::ResidualArgs a{};
    a.stream_in = stream_in;
    a.branch = branch;
    a.stream_out = stream_out;
    a.theta = gate ? nullptr : p;
    a.gate = gate ? p : nullptr;
    a.rows = rows;
    a.width = hidden;
    a.temperature = temperature;
    a.eps = eps;
    return from_cuda(muse::launch_residual_blend(branch_dtype, gate, a, stream), name);
}

}  // namespace

extern "C" {

muse_status muse_residual_blend(const float* stream_in, const void* branch, float* stream_out,
                                muse_dtype branch_dtype, int64_t rows, int64_t hidden, const float* theta,
                                cudaStream_t stream) {
    return residual_entry(stream_in, branch, stream_out, branch_dtype, rows, hidden, theta, false, 1.0f, 0.0f,
                          stream, "muse_residual_blend");
}

muse_status muse_residual(const float* stream_in, const void* branch, float* stream_out, muse_dtype branch_dtype,
                          int64_t rows, int64_t hidden, const float* gate, float temperature, float eps,
                          cudaStream_t stream) {
    return residual_entry(stream_in, branch, stream_out, branch_dtype, rows, hidden, gate, true, temperature, eps,
                          stream, "muse_residual");
}

}  // extern "C"

namespace {

// The backward's row blocks at most, for either branch dtype: its CTAs are
// min(256, vectors per row rounded up to 32) threads, so at most
// min(32, 2048 / threads) of them reside on an SM; the row blocks are those
// resident CTAs over the column blocks, and no more than the row tiles of 4
// (an upper bound: the kernel takes tiles of 8 rows).
int64_t residual_bwd_parts_cap(int64_t rows, int64_t hidden) {
    int64_t cap = 0;
    for (int vec : {8, 4}) {
        const int64_t nvec = hidden / vec;
        if (nvec < 1) continue;
        const int64_t threads = nvec >= 256 ? 256 : (nvec + 31) / 32 * 32;
        const int64_t per_sm = 2048 / threads < 32 ? 2048 / threads : 32;
        const int64_t gy = (nvec + threads - 1) / threads;
        const int64_t gx = (per_sm * (int64_t)muse::sm_count() + gy - 1) / gy;
        if (gx > cap) cap = gx;
    }
    const int64_t tiles = (rows + 3) / 4;
    return tiles < cap ? tiles : cap;
}

muse_status residual_bwd_entry(const float* stream_in, const void* branch, const float* dstream_out,
                               float* dstream_in, void* dbranch, muse_dtype branch_dtype, int64_t rows,
                               int64_t hidden, const float* p, bool gate, float temperature, float eps,
                               float* dparam, void* ws, size_t ws_bytes, cudaStream_t stream, const char* name) {
    if (!valid_dtype(branch_dtype)) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: unknown dtype %d", name, (int)branch_dtype);
    if (rows < 0 || hidden <= 0)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: rows=%lld hidden=%lld", name, (long long)rows, (long long)hidden);
    if (gate && !(finite(temperature) && temperature > 0.0f && finite(eps) && eps >= 0.0f && eps <= 1.0f))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: temperature must be finite and > 0, eps in [0, 1]", name);
    if (!p) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: null %s", name, gate ? "gate" : "theta");
    if (rows == 0) {
        if (dparam) return from_cuda(cudaMemsetAsync(dparam, 0, sizeof(float) * (size_t)hidden, stream), name);
        return MUSE_OK;
    }
    if (!stream_in || !branch || !dstream_out || !dstream_in || !dbranch)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: null tensor", name);
    const int64_t es = elem_size(branch_dtype);
    if (!aligned(stream_in, 16) || !aligned(branch, 16) || !aligned(dstream_out, 16) || !aligned(dstream_in, 16) ||
        !aligned(dbranch, 16) || !aligned(p, 16) || (dparam && !aligned(dparam, 16)) || (hidden * es) % 16)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: pointers and row widths must be 16-byte multiples", name);
    if (hidden / vec_elems(branch_dtype) > (int64_t)65535 * 256)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: rows of more than %d 16-byte vectors", name, 65535 * 256);
    const size_t need = (size_t)residual_bwd_parts_cap(rows, hidden) * (size_t)hidden * sizeof(float);
    if (dparam) {
        muse_status st = bwd_workspace_check(name, need, ws, ws_bytes, true);
        if (st != MUSE_OK) return st;
    }
    const Span sh = span(stream_in, rows, hidden, hidden, 4), sdo = span(dstream_out, rows, hidden, hidden, 4);
    const Span sb = span(branch, rows, hidden, hidden, es), sdb = span(dbranch, rows, hidden, hidden, es);
    const Span sdi = span(dstream_in, rows, hidden, hidden, 4), sp = span(p, 1, hidden, hidden, 4);
    const Span sdp = span(dparam, dparam ? 1 : 0, hidden, hidden, 4);
    const Span sws = span(ws, dparam ? 1 : 0, (int64_t)ws_bytes, (int64_t)ws_bytes, 1);
    bool bad = bad_alias(sdi, sdo, true) || any_overlap(sdi, {sh, sb, sdb, sp, sdp, sws});
    bad = bad || bad_alias(sdb, sb, true) || any_overlap(sdb, {sh, sdo, sp, sdp, sws});
    bad = bad || any_overlap(sdp, {sh, sdo, sb, sp, sws}) || any_overlap(sws, {sh, sdo, sb, sp});
    if (bad) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: an output or the workspace overlaps another tensor", name);
    muse::ResidualArgs a{};
    a.stream_in = stream_in;
    a.branch = branch;
    a.stream_out = dstream_in;
    a.theta = gate ? nullptr : p;
    a.gate = gate ? p : nullptr;
    a.rows = rows;
    a.width = hidden;
    a.temperature = temperature;
    a.eps = eps;
    a.dy = dstream_out;
    a.dbranch = dbranch;
    a.part = dparam ? static_cast<float*>(ws) : nullptr;
    if (dparam) {
        int64_t gx = 0;
        muse_status st = from_cuda(muse::launch_residual_blend_bwd(branch_dtype, gate, a, dparam, stream, &gx), name);
        if (st != MUSE_OK) return st;
        if ((size_t)gx * (size_t)hidden * sizeof(float) > need)
            return fail(MUSE_ERR_UNSUPPORTED, "%s: the grid's partial rows exceed the workspace bound", name);
    }
    return from_cuda(muse::launch_residual_blend_bwd(branch_dtype, gate, a, dparam, stream), name);
}

}  // namespace

extern "C" {

size_t muse_residual_backward_workspace_bytes(int64_t rows, int64_t hidden) {
    if (rows <= 0 || hidden <= 0 || hidden > (int64_t)1 << 30) return 0;
    return (size_t)residual_bwd_parts_cap(rows, hidden) * (size_t)hidden * sizeof(float);
}

muse_status muse_residual_blend_backward(const float* stream_in, const void* branch, const float* dstream_out,
                                         float* dstream_in, void* dbranch, muse_dtype branch_dtype, int64_t rows,
                                         int64_t hidden, const float* theta, float* dtheta, void* workspace,
                                         size_t workspace_bytes, cudaStream_t stream) {
    return residual_bwd_entry(stream_in, branch, dstream_out, dstream_in, dbranch, branch_dtype, rows, hidden,
                              theta, false, 1.0f, 0.0f, dtheta, workspace, workspace_bytes, stream,
                              "muse_residual_blend_backward");
}

muse_status muse_residual_backward(const float* stream_in, const void* branch, const float* dstream_out,
                                   float* dstream_in, void* dbranch, muse_dtype branch_dtype, int64_t rows,
                                   int64_t hidden, const float* gate, float temperature, float eps, float* dgate,
                                   void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    return residual_bwd_entry(stream_in, branch, dstream_out, dstream_in, dbranch, branch_dtype, rows, hidden,
                              gate, true, temperature, eps, dgate, workspace, workspace_bytes, stream,
                              "muse_residual_backward");
}

muse_status muse_residual_gate_angles(const float* gate, float* theta, int64_t hidden, float temperature,
                                      float eps, cudaStream_t stream) {
    const char* name = "muse_residual_gate_angles";
    if (hidden <= 0) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: hidden=%lld", name, (long long)hidden);
    if (!(finite(temperature) && temperature > 0.0f && finite(eps) && eps >= 0.0f && eps <= 1.0f))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: temperature must be finite and > 0, eps in [0, 1]", name);
    if (!gate || !theta) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: null gate or theta", name);
    if (!aligned(gate, 4) || !aligned(theta, 4))
        return fail(MUSE_ERR_UNSUPPORTED, "%s: gate / theta not 4-byte aligned", name);
    if (overlap(span(theta, 1, hidden, hidden, 4), span(gate, 1, hidden, hidden, 4)) && theta != gate)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: theta partially overlaps gate", name);
    if (hidden > ((int64_t)1 << 31) - 256) return fail(MUSE_ERR_UNSUPPORTED, "%s: hidden too large", name);
    muse::ResidualArgs a{};
    a.gate = gate;
    a.width = hidden;
    a.temperature = temperature;
    a.eps = eps;
    return from_cuda(muse::launch_residual_gate_angles(a, theta, stream), name);
}

size_t muse_norm_backward_workspace_bytes(int64_t rows, int64_t hidden) {
    if (rows <= 0 || hidden <= 0 || hidden > (int64_t)1 << 30) return 0;
    return muse::row_bwd_workspace_bytes(rows, (int32_t)hidden);
}

muse_status muse_rms_norm_backward(const void* x, const void* dy, void* dx, muse_dtype dtype,
                                   int64_t rows, int64_t hidden, int64_t x_row_stride,
                                   int64_t dy_row_stride, int64_t dx_row_stride,
                                   const float* gain, float gain_offset, float eps, float* dgain,
                                   void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    return row_bwd_entry(false, x, dy, dx, dtype, rows, hidden, x_row_stride, dy_row_stride,
                         dx_row_stride, gain, gain_offset, eps, dgain, workspace, workspace_bytes,
                         stream, "muse_rms_norm_backward");
}

muse_status muse_rms_norm_backward_noalloc(const void* x, const void* dy, void* dx, muse_dtype dtype,
                                           int64_t rows, int64_t hidden, int64_t x_row_stride,
                                           int64_t dy_row_stride, int64_t dx_row_stride,
                                           const float* gain, float gain_offset, float eps,
                                           float* dgain, cudaStream_t stream) {
    return row_bwd_entry(false, x, dy, dx, dtype, rows, hidden, x_row_stride, dy_row_stride,
                         dx_row_stride, gain, gain_offset, eps, dgain, nullptr, 0, stream,
                         "muse_rms_norm_backward_noalloc", true);
}

muse_status muse_input_scale_norm_backward(const void* x, const void* dy, void* dx,
                                           muse_dtype dtype, int64_t rows, int64_t hidden,
                                           int64_t x_row_stride, int64_t dy_row_stride,
                                           int64_t dx_row_stride, const float* gain,
                                           float gain_offset, float eps, float* dgain,
                                           void* workspace, size_t workspace_bytes,
                                           cudaStream_t stream) {
    return row_bwd_entry(true, x, dy, dx, dtype, rows, hidden, x_row_stride, dy_row_stride,
                         dx_row_stride, gain, gain_offset, eps, dgain, workspace, workspace_bytes,
                         stream, "muse_input_scale_norm_backward");
}

muse_status muse_norm_residual_backward(const float* stream_in, const void* branch,
                                        const float* dstream_out, float* dstream_in,
                                        void* dbranch, muse_dtype branch_dtype, int64_t rows,
                                        int64_t hidden, const float* gain, float gain_offset,
                                        const float* theta, int input_scale, float norm_eps,
                                        float* dgain, float* dtheta, void* workspace,
                                        size_t workspace_bytes, cudaStream_t stream) {
    const char* name = "muse_norm_residual_backward";
    if (!valid_dtype(branch_dtype)) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: unknown dtype %d", name, (int)branch_dtype);
    if (rows < 0 || hidden <= 0)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: rows=%lld hidden=%lld", name, (long long)rows, (long long)hidden);
    if (!finite(norm_eps) || norm_eps < 0.0f || !finite(gain_offset))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: norm_eps must be finite and >= 0, gain_offset finite", name);
    if (dgain && !gain) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: dgain requested without a gain", name);
    if (rows == 0) {
        cudaError_t e = cudaSuccess;
        if (dgain) e = cudaMemsetAsync(dgain, 0, sizeof(float) * (size_t)hidden, stream);
        if (e == cudaSuccess && dtheta) e = cudaMemsetAsync(dtheta, 0, sizeof(float) * (size_t)hidden, stream);
        return from_cuda(e, name);
    }
    if (!stream_in || !branch || !dstream_out || !dstream_in || !dbranch || !theta)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: null tensor", name);
    const int64_t es = elem_size(branch_dtype);
    if (!aligned(stream_in, 16) || !aligned(branch, 16) || !aligned(dstream_out, 16) || !aligned(dstream_in, 16) ||
        !aligned(dbranch, 16) || (hidden * es) % 16)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: pointers and row widths must be 16-byte multiples", name);
    if (!aligned(theta, 16) || (gain && !aligned(gain, 16)) || (dgain && !aligned(dgain, 16)) ||
        (dtheta && !aligned(dtheta, 16)))
        return fail(MUSE_ERR_UNSUPPORTED, "%s: theta / gain / dgain / dtheta not 16-byte aligned", name);
    if (hidden / vec_elems(branch_dtype) > muse::kBwdMaxVectors)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: rows of more than %d 16-byte vectors", name, muse::kBwdMaxVectors);
    muse_status st = bwd_workspace_check(name, muse::row_bwd_workspace_bytes(rows, (int32_t)hidden),
                                         workspace, workspace_bytes, dgain || dtheta);
    if (st != MUSE_OK) return st;
    const Span sh = span(stream_in, rows, hidden, hidden, 4), sdo = span(dstream_out, rows, hidden, hidden, 4);
    const Span sb = span(branch, rows, hidden, hidden, es), sdb = span(dbranch, rows, hidden, hidden, es);
    const Span sdi = span(dstream_in, rows, hidden, hidden, 4), sth = span(theta, 1, hidden, hidden, 4);
    const Span sg = span(gain, gain ? 1 : 0, hidden, hidden, 4), sdg = span(dgain, dgain ? 1 : 0, hidden, hidden, 4);
    const Span sdt = span(dtheta, dtheta ? 1 : 0, hidden, hidden, 4);
    const Span sws = span(workspace, (dgain || dtheta) ? 1 : 0, (int64_t)workspace_bytes, (int64_t)workspace_bytes, 1);
    bool bad = bad_alias(sdi, sdo, true) || any_overlap(sdi, {sh, sb, sdb, sth, sg, sdg, sdt, sws});
    bad = bad || bad_alias(sdb, sb, true) || any_overlap(sdb, {sh, sdo, sth, sg, sdg, sdt, sws});
    bad = bad || any_overlap(sdg, {sh, sdo, sb, sth, sg, sdt, sws}) || any_overlap(sdt, {sh, sdo, sb, sth, sg, sws});
    bad = bad || any_overlap(sws, {sh, sdo, sb, sth, sg});
    if (bad) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: an output or the workspace overlaps another tensor", name);
    muse::RowBwdArgs a{};
    a.x = branch;
    a.dy = dstream_out;
    a.stream_in = stream_in;
    a.dx = dbranch;
    a.dstream_in = dstream_in;
    a.gain = gain;
    a.theta = theta;
    a.rows = rows;
    a.x_stride = a.dy_stride = a.dx_stride = hidden;
    a.width = (int32_t)hidden;
    a.gain_offset = gain_offset;
    a.eps = norm_eps;
    if (dgain || dtheta) {
        const int64_t cap = (int64_t)(muse::row_bwd_workspace_bytes(rows, (int32_t)hidden) / 2 / sizeof(float));
        a.part_gain = static_cast<float*>(workspace);
        a.part_theta = static_cast<float*>(workspace) + cap;
    }
    const muse::BwdOp op = input_scale ? muse::BwdOp::kResidualIS : muse::BwdOp::kResidual;
    return from_cuda(muse::launch_row_bwd(branch_dtype, op, a, dgain, dtheta, stream), name);
}

muse_status muse_output_norm_gate_backward(const void* o, const void* gate, const void* dy, void* d_o,
                                           void* dgate, muse_dtype dtype, int64_t tokens,
                                           int32_t heads, int32_t head_dim, int32_t norm_group,
                                           float eps, cudaStream_t stream) {
    const char* name = "muse_output_norm_gate_backward";
    if (!valid_dtype(dtype)) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: unknown dtype %d", name, (int)dtype);
    if (tokens < 0 || heads <= 0 || head_dim <= 0)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: tokens=%lld heads=%d head_dim=%d", name, (long long)tokens, heads, head_dim);
    const int64_t width = (int64_t)heads * head_dim;
    if (norm_group != head_dim && norm_group != width)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: norm_group=%d must be head_dim or heads*head_dim", name, norm_group);
    if (!finite(eps) || eps < 0.0f) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: eps must be finite and >= 0", name);
    if (tokens == 0) return MUSE_OK;
    if (!o || !gate || !dy || !d_o || !dgate) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: null tensor", name);
    const int64_t es = elem_size(dtype);
    if (!aligned(o, 16) || !aligned(gate, 16) || !aligned(dy, 16) || !aligned(d_o, 16) || !aligned(dgate, 16) ||
        (head_dim * es) % 16)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: pointers and head_dim must be 16-byte multiples", name);
    if (norm_group * es > MUSE_MAX_ROW_BYTES)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: norm group of %lld bytes exceeds %d", name, (long long)(norm_group * es), MUSE_MAX_ROW_BYTES);
    const Span so = span(o, tokens, width, width, es), sg = span(gate, tokens, width, width, es);
    const Span sdy = span(dy, tokens, width, width, es), sdo = span(d_o, tokens, width, width, es);
    const Span sdg = span(dgate, tokens, width, width, es);
    // do may coincide with o or dy, dgate with gate or dy; never with each other
    bool bad = (!same_span(sdo, so) && !same_span(sdo, sdy) && any_overlap(sdo, {so, sdy})) || overlap(sdo, sg);
    bad = bad || (!same_span(sdg, sg) && !same_span(sdg, sdy) && any_overlap(sdg, {sg, sdy})) || overlap(sdg, so);
    bad = bad || overlap(sdo, sdg);
    if (bad) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: an output partially overlaps an input", name);
    muse::GateBwdArgs a{};
    a.o = o;
    a.gate = gate;
    a.dy = dy;
    a.d_o = d_o;
    a.dgate = dgate;
    a.rows = tokens * (width / norm_group);
    a.width = norm_group;
    a.eps = eps;
    return from_cuda(muse::launch_gate_bwd(dtype, a, stream), name);
}

muse_status muse_qk_norm_rope_backward(const void* q, const void* k, const void* dq_out,
                                       const void* dk_out, void* dq, void* dk, muse_dtype dtype,
                                       muse_layout layout, int64_t batch, int64_t seqlen,
                                       const int32_t* cu_seqlens, int32_t num_seqs,
                                       int64_t total_tokens, const int32_t* positions, int32_t hq,
                                       int32_t hkv, int32_t head_dim, int64_t q_tok_stride,
                                       int64_t k_tok_stride, int64_t dq_out_tok_stride,
                                       int64_t dk_out_tok_stride, int64_t dq_tok_stride,
                                       int64_t dk_tok_stride, float eps, float query_scale,
                                       int use_rope, int upcast_rope, float rope_base,
                                       cudaStream_t stream) {
    const char* name = "muse_qk_norm_rope_backward";
    if (!valid_dtype(dtype)) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: unknown dtype %d", name, (int)dtype);
    if (layout != MUSE_LAYOUT_BSHD && layout != MUSE_LAYOUT_THD)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: unknown layout %d", name, (int)layout);
    int64_t tokens;
    if (layout == MUSE_LAYOUT_BSHD) {
        if (batch < 0 || seqlen <= 0)
            return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: batch=%lld seqlen=%lld", name, (long long)batch, (long long)seqlen);
        tokens = batch * seqlen;
    } else {
        if (total_tokens < 0) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: total_tokens < 0", name);
        tokens = total_tokens;
    }
    if (hkv <= 0 || hq <= 0 || hq % hkv)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: hq=%d must be a positive multiple of hkv=%d", name, hq, hkv);
    if (head_dim <= 0 || (head_dim & 1))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: head_dim=%d must be positive and even", name, head_dim);
    if (!finite(eps) || eps < 0.0f || !finite(query_scale))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: eps must be finite and >= 0, query_scale finite", name);
    if (use_rope && !(finite(rope_base) && rope_base > 0.0f))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: rope_base must be finite and > 0", name);
    const int64_t qw = (int64_t)hq * head_dim, kw = (int64_t)hkv * head_dim;
    if (q_tok_stride < qw || dq_out_tok_stride < qw || dq_tok_stride < qw || k_tok_stride < kw ||
        dk_out_tok_stride < kw || dk_tok_stride < kw)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: token strides must cover all heads", name);
    const bool derive = use_rope && !positions;
    if (tokens > 0 && derive && layout == MUSE_LAYOUT_THD && (!cu_seqlens || num_seqs < 1))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: THD without positions needs cu_seqlens and num_seqs >= 1", name);
    if (tokens == 0) return MUSE_OK;
    if (!q || !k || !dq_out || !dk_out || !dq || !dk) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: null tensor", name);
    const int64_t es = elem_size(dtype);
    const void* ptrs[6] = {q, k, dq_out, dk_out, dq, dk};
    for (const void* p : ptrs)
        if (!aligned(p, 16)) return fail(MUSE_ERR_UNSUPPORTED, "%s: pointers must be 16-byte aligned", name);
    const int64_t strides[6] = {q_tok_stride, k_tok_stride, dq_out_tok_stride, dk_out_tok_stride, dq_tok_stride, dk_tok_stride};
    for (int64_t st : strides)
        if ((st * es) % 16) return fail(MUSE_ERR_UNSUPPORTED, "%s: strides must be 16-byte multiples", name);
    if ((head_dim * es) % 16 || head_dim / vec_elems(dtype) > 32 || head_dim / 2 > muse::kMaxHalfDim)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: head_dim=%d must be 16-byte multiple of at most 512 bytes", name, head_dim);
    if ((positions && !aligned(positions, 4)) || (cu_seqlens && !aligned(cu_seqlens, 4)))
        return fail(MUSE_ERR_UNSUPPORTED, "%s: positions / cu_seqlens not 4-byte aligned", name);
    const Span sq = span(q, tokens, qw, q_tok_stride, es), sk = span(k, tokens, kw, k_tok_stride, es);
    const Span sgq = span(dq_out, tokens, qw, dq_out_tok_stride, es), sgk = span(dk_out, tokens, kw, dk_out_tok_stride, es);
    const Span sdq = span(dq, tokens, qw, dq_tok_stride, es), sdk = span(dk, tokens, kw, dk_tok_stride, es);
    // dq may coincide with q or dq_out, dk with k or dk_out
    bool bad = (!same_span(sdq, sq) && !same_span(sdq, sgq) && any_overlap(sdq, {sq, sgq})) || any_overlap(sdq, {sk, sgk, sdk});
    bad = bad || (!same_span(sdk, sk) && !same_span(sdk, sgk) && any_overlap(sdk, {sk, sgk})) || any_overlap(sdk, {sq, sgq});
    if (use_rope && positions) {
        const Span sp = span(positions, 1, tokens, tokens, 4);
        bad = bad || overlap(sdq, sp) || overlap(sdk, sp);
    }
    if (derive && layout == MUSE_LAYOUT_THD) {
        const Span sc = span(cu_seqlens, 1, (int64_t)num_seqs + 1, (int64_t)num_seqs + 1, 4);
        bad = bad || overlap(sdq, sc) || overlap(sdk, sc);
    }
    if (bad) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: an output partially overlaps an input", name);
    muse::QkBwdArgs A{};
    muse::QkArgs& a = A.f;
    a.q = q;
    a.k = k;
    a.q_out = dq;
    a.k_out = dk;
    a.positions = positions;
    a.cu_seqlens = cu_seqlens;
    a.tokens = tokens;
    a.seqlen = layout == MUSE_LAYOUT_BSHD ? seqlen : 1;
    a.q_stride = q_tok_stride;
    a.k_stride = k_tok_stride;
    a.q_out_stride = dq_tok_stride;
    a.k_out_stride = dk_tok_stride;
    a.num_seqs = num_seqs;
    a.hq = hq;
    a.hkv = hkv;
    a.head_dim = head_dim;
    a.pos_mode = positions ? 0 : (layout == MUSE_LAYOUT_BSHD ? 1 : 2);
    a.eps = eps;
    a.query_scale = query_scale;
    if (use_rope)
        for (int i = 0; i < head_dim / 2; ++i)
            a.inv_freq[i] = (float)std::pow((double)rope_base, -(2.0 * i) / (double)head_dim);
    A.gq = dq_out;
    A.gk = dk_out;
    A.gq_stride = dq_out_tok_stride;
    A.gk_stride = dk_out_tok_stride;
    return from_cuda(muse::launch_qk_bwd(dtype, use_rope, upcast_rope, A, stream), name);
}

muse_status muse_rms_norm_grouped(const void* x, void* y, muse_dtype dtype, int64_t rows, int64_t hidden,
                                  int64_t x_row_stride, int64_t y_row_stride, const float* gains,
                                  float gain_offset, const int32_t* group_offsets, int32_t num_groups,
                                  float eps, cudaStream_t stream) {
    const char* name = "muse_rms_norm_grouped";
    if (!valid_dtype(dtype)) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: unknown dtype %d", name, (int)dtype);
    if (rows < 0 || hidden <= 0 || num_groups < 1)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: rows=%lld hidden=%lld num_groups=%d", name, (long long)rows,
                    (long long)hidden, num_groups);
    if (!finite(eps) || eps < 0.0f || !finite(gain_offset))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: eps must be finite and >= 0, gain_offset finite", name);
    if (x_row_stride < hidden || y_row_stride < hidden)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: row strides must be >= hidden", name);
    if (rows == 0) return MUSE_OK;
    if (!x || !y || !gains || !group_offsets)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: null x, y, gains or group_offsets", name);
    const int64_t es = elem_size(dtype);
    if (!aligned(x, 16) || !aligned(y, 16) || !aligned(gains, 16) || (hidden * es) % 16 ||
        (x_row_stride * es) % 16 || (y_row_stride * es) % 16)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: pointers, row widths and strides must be 16-byte multiples", name);
    if (!aligned(group_offsets, 4)) return fail(MUSE_ERR_UNSUPPORTED, "%s: group_offsets not 4-byte aligned", name);
    if (hidden / vec_elems(dtype) > 1024)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: rows of more than 1024 16-byte vectors", name);
    const Span sx = span(x, rows, hidden, x_row_stride, es), sy = span(y, rows, hidden, y_row_stride, es);
    const Span sg = span(gains, num_groups, hidden, hidden, 4);
    const Span so = span(group_offsets, 1, (int64_t)num_groups + 1, (int64_t)num_groups + 1, 4);
    if (bad_alias(sy, sx, true) || any_overlap(sy, {sg, so}))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: output partially overlaps an input", name);
    muse::RowArgs a{};
    a.x = x;
    a.y = y;
    a.gain = gains;
    a.rows = rows;
    a.x_stride = x_row_stride;
    a.y_stride = y_row_stride;
    a.width = (int32_t)hidden;
    a.gain_offset = gain_offset;
    a.eps = eps;
    a.group_offsets = group_offsets;
    a.num_groups = num_groups;
    return from_cuda(muse::launch_row(dtype, muse::RowOp::kRmsGrouped, a, stream), name);
}

muse_status muse_norm_residual_rms_norm(const float* stream_in, const void* branch, float* stream_out,
                                        void* y, muse_dtype branch_dtype, muse_dtype y_dtype,
                                        int64_t rows, int64_t hidden, const float* gain,
                                        float gain_offset, const float* theta, int input_scale,
                                        float norm_eps, const float* next_gain,
                                        float next_gain_offset, float next_eps,
                                        cudaStream_t stream) {
    const char* name = "muse_norm_residual_rms_norm";
    if (!valid_dtype(branch_dtype) || !valid_dtype(y_dtype))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: unknown dtype", name);
    if (rows < 0 || hidden <= 0)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: rows=%lld hidden=%lld", name, (long long)rows, (long long)hidden);
    if (!finite(norm_eps) || norm_eps < 0.0f || !finite(gain_offset) || !finite(next_eps) || next_eps < 0.0f ||
        !finite(next_gain_offset))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: eps values must be finite and >= 0, offsets finite", name);
    if (rows == 0) return MUSE_OK;
    if (!stream_in || !branch || !stream_out || !theta || !y)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: null stream_in/branch/stream_out/theta/y", name);
    const int64_t es = elem_size(branch_dtype), ys = elem_size(y_dtype);
    if (!aligned(stream_in, 16) || !aligned(stream_out, 16) || !aligned(branch, 16) || !aligned(y, 16) ||
        (hidden * es) % 16 || (hidden * ys) % 16)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: pointers and row widths must be 16-byte multiples", name);
    if (!aligned(theta, 16) || (gain && !aligned(gain, 16)) || (next_gain && !aligned(next_gain, 16)))
        return fail(MUSE_ERR_UNSUPPORTED, "%s: theta / gains not 16-byte aligned", name);
    if (hidden / vec_elems(branch_dtype) > 1024)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: rows of more than 1024 16-byte branch vectors", name);
    if (y_dtype != MUSE_DTYPE_F32 && y_dtype != branch_dtype)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: y must be FP32 or in the branch dtype", name);
    const Span sin_ = span(stream_in, rows, hidden, hidden, 4), sout = span(stream_out, rows, hidden, hidden, 4);
    const Span sb = span(branch, rows, hidden, hidden, es), st = span(theta, 1, hidden, hidden, 4);
    const Span sy = span(y, rows, hidden, hidden, ys);
    const Span sg = span(gain, gain ? 1 : 0, hidden, hidden, 4), sg2 = span(next_gain, next_gain ? 1 : 0, hidden, hidden, 4);
    bool bad = bad_alias(sout, sin_, true) || any_overlap(sout, {sb, st, sg, sg2, sy});
    bad = bad || (!same_span(sy, sb) && overlap(sy, sb)) || any_overlap(sy, {sin_, st, sg, sg2});
    if (bad) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: an output partially overlaps an input", name);
    muse::RowArgs a{};
    a.x = branch;
    a.y = y;
    a.stream_in = stream_in;
    a.stream_out = stream_out;
    a.gain = gain;
    a.theta = theta;
    a.rows = rows;
    a.x_stride = hidden;
    a.y_stride = hidden;
    a.s_in_stride = a.s_out_stride = hidden;
    a.width = (int32_t)hidden;
    a.gain_offset = gain_offset;
    a.eps = norm_eps;
    a.gain2 = next_gain;
    a.gain2_offset = next_gain_offset;
    a.eps2 = next_eps;
    a.y_f32 = y_dtype == MUSE_DTYPE_F32 ? 1 : 0;
    const muse::RowOp op = input_scale ? muse::RowOp::kResidualISPre : muse::RowOp::kResidualPre;
    return from_cuda(muse::launch_row(branch_dtype, op, a, stream), name);
}

muse_status muse_residual_blend_rms_norm(const float* stream_in, const void* branch, float* stream_out, void* y,
                                         muse_dtype branch_dtype, muse_dtype y_dtype, int64_t rows, int64_t hidden,
                                         const float* theta, const float* next_gain, float next_gain_offset,
                                         float next_eps, cudaStream_t stream) {
    const char* name = "muse_residual_blend_rms_norm";
    if (!valid_dtype(branch_dtype) || !valid_dtype(y_dtype))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: unknown dtype", name);
    if (rows < 0 || hidden <= 0)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: rows=%lld hidden=%lld", name, (long long)rows, (long long)hidden);
    if (!finite(next_eps) || next_eps < 0.0f || !finite(next_gain_offset))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: next_eps must be finite and >= 0, next_gain_offset finite", name);
    if (rows == 0) return MUSE_OK;
    if (!stream_in || !branch || !stream_out || !theta || !y)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: null stream_in/branch/stream_out/theta/y", name);
    const int64_t es = elem_size(branch_dtype), ys = elem_size(y_dtype);
    if (!aligned(stream_in, 16) || !aligned(stream_out, 16) || !aligned(branch, 16) || !aligned(y, 16) ||
        (hidden * es) % 16 || (hidden * ys) % 16)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: pointers and row widths must be 16-byte multiples", name);
    if (!aligned(theta, 16) || (next_gain && !aligned(next_gain, 16)))
        return fail(MUSE_ERR_UNSUPPORTED, "%s: theta / next_gain not 16-byte aligned", name);
    if (hidden / vec_elems(branch_dtype) > 1024)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: rows of more than 1024 16-byte branch vectors", name);
    if (y_dtype != MUSE_DTYPE_F32 && y_dtype != branch_dtype)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: y must be FP32 or in the branch dtype", name);
    const Span sin_ = span(stream_in, rows, hidden, hidden, 4), sout = span(stream_out, rows, hidden, hidden, 4);
    const Span sb = span(branch, rows, hidden, hidden, es), st = span(theta, 1, hidden, hidden, 4);
    const Span sy = span(y, rows, hidden, hidden, ys);
    const Span sg2 = span(next_gain, next_gain ? 1 : 0, hidden, hidden, 4);
    bool bad = bad_alias(sout, sin_, true) || any_overlap(sout, {sb, st, sg2, sy});
    bad = bad || (!same_span(sy, sb) && overlap(sy, sb)) || any_overlap(sy, {sin_, st, sg2});
    if (bad) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: an output partially overlaps an input", name);
    muse::RowArgs a{};
    a.x = branch;
    a.y = y;
    a.stream_in = stream_in;
    a.stream_out = stream_out;
    a.theta = theta;
    a.rows = rows;
    a.x_stride = hidden;
    a.y_stride = hidden;
    a.s_in_stride = a.s_out_stride = hidden;
    a.width = (int32_t)hidden;
    a.gain2 = next_gain;
    a.gain2_offset = next_gain_offset;
    a.eps2 = next_eps;
    a.y_f32 = y_dtype == MUSE_DTYPE_F32 ? 1 : 0;
    return from_cuda(muse::launch_row(branch_dtype, muse::RowOp::kBlendPre, a, stream), name);
}

muse_status muse_device_error(unsigned int* flags, int clear) {
    if (!flags) return fail(MUSE_ERR_INVALID_ARGUMENT, "muse_device_error: null flags");
    // bit 0: the row pipeline's word, bit 1: the Q/K ring's, bit 2: the row
    // backward's, bit 3: the Q/K backward ring's
    unsigned int row = 0, qk = 0, bwd = 0, qkb = 0;
    cudaError_t e = muse::read_device_error(&row, clear != 0);
    if (e == cudaSuccess) e = muse::read_qk_device_error(&qk, clear != 0);
    if (e == cudaSuccess) e = muse::read_bwd_device_error(&bwd, clear != 0);
    if (e == cudaSuccess) e = muse::read_qk_bwd_device_error(&qkb, clear != 0);
    *flags = (row ? 1u : 0u) | (qk ? 2u : 0u) | (bwd ? 4u : 0u) | (qkb ? 8u : 0u);
    return from_cuda(e, "muse_device_error");
}

muse_status muse_stream_copy(const void* src, void* dst, int64_t bytes, cudaStream_t stream) {
    const char* name = "muse_stream_copy";
    if (bytes < 0) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: bytes=%lld", name, (long long)bytes);
    if (bytes == 0) return MUSE_OK;
    if (!src || !dst) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: null pointer", name);
    if (bytes % 16 || !aligned(src, 16) || !aligned(dst, 16))
        return fail(MUSE_ERR_UNSUPPORTED, "%s: pointers and size must be 16-byte multiples", name);
    if (overlap(span(src, 1, bytes, bytes, 1), span(dst, 1, bytes, bytes, 1)))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: ranges overlap", name);
    return from_cuda(muse::launch_copy(src, dst, bytes, stream), name);
}

muse_status muse_vision_rope(const void* q, const void* k, void* q_out, void* k_out, muse_dtype dtype,
                             int64_t tokens, int32_t hq, int32_t hk, int32_t head_dim,
                             int64_t q_tok_stride, int64_t k_tok_stride, int64_t q_out_tok_stride,
                             int64_t k_out_tok_stride, const float* freqs, cudaStream_t stream) {
    const char* name = "muse_vision_rope";
    if (!valid_dtype(dtype)) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: unknown dtype %d", name, (int)dtype);
    if (tokens < 0 || hq <= 0 || hk <= 0 || head_dim <= 0 || (head_dim & 1))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: tokens=%lld hq=%d hk=%d head_dim=%d", name,
                    (long long)tokens, hq, hk, head_dim);
    const int64_t qw = (int64_t)hq * head_dim, kw = (int64_t)hk * head_dim;
    if (q_tok_stride < qw || q_out_tok_stride < qw || k_tok_stride < kw || k_out_tok_stride < kw)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: token strides must cover all heads", name);
    if (tokens == 0) return MUSE_OK;
    if (!q || !k || !q_out || !k_out || !freqs)
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: null q, k, q_out, k_out or freqs", name);
    const int64_t es = elem_size(dtype);
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(q_out, 16) || !aligned(k_out, 16) || !aligned(freqs, 16) ||
        (head_dim * es) % 16 || (q_tok_stride * es) % 16 || (k_tok_stride * es) % 16 ||
        (q_out_tok_stride * es) % 16 || (k_out_tok_stride * es) % 16)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: pointers, head_dim and strides must be 16-byte multiples", name);
    if ((qw + kw) / vec_elems(dtype) > (int64_t)1 << 30)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: token rows too wide", name);
    if (head_dim * es > 512)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: head_dim=%d exceeds 512 bytes per head", name, head_dim);
    const Span sq = span(q, tokens, qw, q_tok_stride, es), sk = span(k, tokens, kw, k_tok_stride, es);
    const Span sqo = span(q_out, tokens, qw, q_out_tok_stride, es);
    const Span sko = span(k_out, tokens, kw, k_out_tok_stride, es);
    const Span sf = span(freqs, 1, tokens * head_dim, tokens * head_dim, 4);
    if (bad_alias(sqo, sq, true) || bad_alias(sqo, sk, false) || bad_alias(sqo, sko, false) ||
        bad_alias(sko, sk, true) || bad_alias(sko, sq, false) || bad_alias(sqo, sf, false) ||
        bad_alias(sko, sf, false))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: output partially overlaps an input", name);
    muse::VisionRopeArgs a{};
    a.q = q;
    a.k = k;
    a.q_out = q_out;
    a.k_out = k_out;
    a.freqs = freqs;
    a.tokens = tokens;
    a.q_stride = q_tok_stride;
    a.k_stride = k_tok_stride;
    a.q_out_stride = q_out_tok_stride;
    a.k_out_stride = k_out_tok_stride;
    a.hq = hq;
    a.hk = hk;
    a.head_dim = head_dim;
    return from_cuda(muse::launch_vision_rope(dtype, a, stream), name);
}

muse_status muse_vision_rope_frequencies(float* out, int32_t head_dim, int32_t grid_h, int32_t grid_w,
                                         float theta, cudaStream_t stream) {
    const char* name = "muse_vision_rope_frequencies";
    if (head_dim <= 0 || (head_dim & 3) || grid_h < 0 || grid_w < 0 || !(finite(theta) && theta > 0.0f))
        return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: head_dim=%d (a positive multiple of 4), grid %dx%d, theta > 0",
                    name, head_dim, grid_h, grid_w);
    if (head_dim / 4 > muse::kMaxHalfDim)
        return fail(MUSE_ERR_UNSUPPORTED, "%s: head_dim=%d above %d", name, head_dim, 4 * muse::kMaxHalfDim);
    if ((int64_t)grid_h * grid_w == 0) return MUSE_OK;
    if (!out) return fail(MUSE_ERR_INVALID_ARGUMENT, "%s: null out", name);
    if (!aligned(out, 8)) return fail(MUSE_ERR_UNSUPPORTED, "%s: out not 8-byte aligned", name);
    muse::VisionFreqArgs a{};
    a.out = out;
    a.head_dim = head_dim;
    a.grid_h = grid_h;
    a.grid_w = grid_w;
    // frequencies over half the head: theta^(-2j/(head_dim/2)), rounded to FP32
    for (int j = 0; j < head_dim / 4; ++j)
        a.inv_freq[j] = (float)std::pow((double)theta, -(2.0 * j) / (double)(head_dim / 2));
    return from_cuda(muse::launch_vision_rope_frequencies(a, stream), name);
}

}  // extern "C"
