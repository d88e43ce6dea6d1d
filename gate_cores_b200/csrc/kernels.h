// Internal launch interface between the C ABI (api.cu) and the kernel files.
// Host-side only; arguments arrive here already validated.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace muse {

enum class RowOp : int {
    kRms = 0,          // core 1: y = cast((x r) w)
    kInputScale = 1,   // core 2: z = x w, y = cast(z r(z))
    kNormGate = 2,     // core 4, one norm per token row: y = cast(o r sigmoid(g))
    kResidual = 3,     // core 5, gain after the norm
    kResidualIS = 4,   // core 5, gain before the norm
    kResidualPre = 5,    // core 5 (gain after) + the next sublayer's RMS pre-norm of the new stream
    kResidualISPre = 6,  // core 5 (gain before) + the next sublayer's RMS pre-norm
    kRmsGrouped = 7,     // core 1 with per-expert gains: rows of group g use gain row g
    kBlendPre = 8,       // _residual_core (angle form, no branch norm) + the next sublayer's RMS pre-norm
};

// One row = one token's `width` elements.  Strides in elements.
struct RowArgs {
    const void* x;          // x (cores 1, 2), o (core 4), branch (core 5)
    void* y;                // output rows (cores 1, 2, 4)
    const void* gate;       // core 4
    const float* stream_in; // core 5
    float* stream_out;      // core 5
    const float* gain;      // may be null
    const float* theta;     // core 5
    const float* cos_sin;   // core 5: [cos(theta) | sin(theta)] table, or null
    int64_t rows;
    int64_t x_stride, y_stride, gate_stride, s_in_stride, s_out_stride;
    int32_t width;
    int32_t rows_per_cta;   // set by the launcher (register-staged row kernels)
    float gain_offset;
    float eps;
    // kResidualPre / kResidualISPre / kBlendPre: y = cast((h' r(h')) (gain2 + gain2_offset))
    // into `y` (row stride y_stride), FP32 when y_f32 else the branch dtype
    const float* gain2;     // may be null
    float gain2_offset;
    float eps2;
    int32_t y_f32;
    // kRmsGrouped: gain is [num_groups, width]; rows [offsets[g], offsets[g+1]) use row g
    const int32_t* group_offsets;
    int32_t num_groups;
    // Bounded-wait probe (0 / unset in every ordinary call): spin_limit > 0
    // replaces the default poll limit of every mbarrier wait; with
    // probe_stall != 0 the producer never signals the stage of row stall_row
    // (and issues nothing after it), so that row's wait runs out.
    uint32_t spin_limit;
    int32_t probe_stall;
    int64_t stall_row;
};

// Many short rows (one attention head each), contiguous: core 4 per head.
struct HeadGateArgs {
    const void* o;
    const void* gate;
    void* y;
    int64_t rows;     // tokens * heads
    int32_t width;    // head_dim
    float eps;
};

// Backward of the row-wide cores (cores 1, 2, 5): one row per token.
enum class BwdOp : int {
    kRms = 0,          // core 1
    kInputScale = 1,   // core 2
    kResidual = 2,     // core 5, gain after the norm
    kResidualIS = 3,   // core 5, gain before the norm
};

struct RowBwdArgs {
    const void* x;          // x (cores 1, 2) or the branch (core 5)
    const void* dy;         // dL/dy (cores 1, 2; x's dtype) or dL/dstream_out (core 5; FP32)
    const float* stream_in; // core 5: the forward's stream h
    void* dx;               // dL/dx (cores 1, 2) or dL/dbranch (core 5), x's dtype
    float* dstream_in;      // core 5: dL/dh
    const float* gain;      // may be null (no gain gradient then)
    const float* theta;     // core 5
    float* part_gain;       // [grid][width] per-CTA partial gain gradients, or null
    float* part_theta;      // core 5: [grid][width] per-CTA partial theta gradients
    int64_t rows;
    int64_t x_stride, dy_stride, dx_stride;  // elements; core 5 rows are contiguous
    int32_t width;
    float gain_offset;
    float eps;
};

// Largest row (in 16-byte vectors) the row backward handles, and the
// workspace it needs for `rows` rows of `width` elements.
constexpr int kBwdMaxVectors = 1024;
size_t row_bwd_workspace_bytes(int64_t rows, int32_t width);
// Scratch of the allocation-free core 1 backward: bytes its gain partials need,
// the fixed capacity, and the device address of the fixed array (looked up
// once per device, then cached).
size_t row_bwd_gain_scratch_bytes(int64_t rows, int32_t width);
constexpr size_t kNoAllocScratchBytes = (size_t)16 << 20;
cudaError_t noalloc_scratch(void** ptr);
// The grid a row backward launch of these arguments uses on the current
// device (nothing is launched); its gain partials take grid * width floats.
cudaError_t row_bwd_launch_grid(int dtype, BwdOp op, const RowBwdArgs& a, int64_t* grid);

constexpr int kMaxHalfDim = 128;  // head_dim <= 256

struct QkArgs {
    const void* q;
    const void* k;
    void* q_out;
    void* k_out;
    const int32_t* positions;   // explicit positions or null
    const int32_t* cu_seqlens;  // THD document boundaries (positions == null)
    int64_t tokens;
    int64_t seqlen;             // BSHD: positions derive as t mod seqlen
    int64_t q_stride, k_stride, q_out_stride, k_out_stride;  // elements per token
    int32_t num_seqs;
    int32_t hq, hkv, head_dim;
    int32_t split;              // forward: warps sharing one token's head steps (1, 2, 4, 8; set by the launcher)
    int32_t pos_mode;           // 0 explicit, 1 BSHD derived, 2 THD derived
    float eps;
    float query_scale;
    float inv_freq[kMaxHalfDim];
};

// Backward of core 4 over contiguous groups of `width` elements (one head or
// one token each): do and dgate from o, gate and dy.
struct GateBwdArgs {
    const void* o;
    const void* gate;
    const void* dy;
    void* d_o;
    void* dgate;
    int64_t rows;     // groups
    int32_t width;    // elements per group
    float eps;
};
cudaError_t launch_gate_bwd(int dtype, const GateBwdArgs& a, cudaStream_t s);

// Backward of core 3 (FP32 rotation or none): f holds the forward's inputs
// (q, k, positions, layout, sizes, eps, query_scale, inv_freq) and, as
// q_out / k_out, the gradient outputs dq / dk with their token strides; gq /
// gk are the incoming gradients dL/dq_out, dL/dk_out.
struct QkBwdArgs {
    QkArgs f;
    const void* gq;
    const void* gk;
    int64_t gq_stride, gk_stride;
};
cudaError_t launch_qk_bwd(int dtype, int use_rope, int upcast_rope, const QkBwdArgs& a, cudaStream_t s);

// Vision 2-D RoPE: Q [tokens, hq, head_dim] and K [tokens, hk, head_dim] with
// per-token strides, rotated by the table freqs [tokens, head_dim/2, 2]
// (cos, sin per pair, contiguous).
struct VisionRopeArgs {
    const void* q;
    const void* k;
    void* q_out;
    void* k_out;
    const float* freqs;
    int64_t tokens;
    int64_t q_stride, k_stride, q_out_stride, k_out_stride;  // elements per token
    int32_t hq, hk, head_dim;
};
// The table of one row-major grid_h x grid_w patch grid: out
// [grid_h * grid_w, head_dim/2, 2]; inv_freq[j], j < head_dim/4.
struct VisionFreqArgs {
    float* out;
    int32_t head_dim, grid_h, grid_w;
    float inv_freq[kMaxHalfDim];
};
cudaError_t launch_vision_rope(int dtype, const VisionRopeArgs& a, cudaStream_t s);
cudaError_t launch_vision_rope_frequencies(const VisionFreqArgs& a, cudaStream_t s);
cudaError_t read_qk_bwd_device_error(unsigned int* out, bool clear);

// _residual_core: stream_out = c * stream_in + s * f32(branch) per channel,
// (c, s) = (cos, sin) of theta, or from the learned gate (gate != null):
// c^2 = max(sigmoid(gate / temperature), eps), s^2 = 1 - c^2.  Rows contiguous.
struct ResidualArgs {
    const float* stream_in;
    const void* branch;
    float* stream_out;      // forward: the new stream; backward: dL/dstream_in
    const float* theta;     // angle form
    const float* gate;      // gate form
    int64_t rows;
    int64_t width;
    float temperature;
    float eps;
    // backward only
    const float* dy;        // dL/dstream_out, FP32 [rows, width]
    void* dbranch;          // dL/dbranch, branch dtype
    float* part;            // [row blocks][width] partial angle / gate gradients (workspace)
};
cudaError_t launch_residual_blend(int dtype, bool gate, const ResidualArgs& a, cudaStream_t s);
// Backward; dparam (dtheta or dgate, [width]) may be null.  With plan_gx the
// row-block count of the grid (the partial rows the workspace must hold) is
// returned and nothing is launched.
cudaError_t launch_residual_blend_bwd(int dtype, bool gate, const ResidualArgs& a, float* dparam,
                                      cudaStream_t s, int64_t* plan_gx = nullptr);
// Deterministic column sums of nparts partial rows of width floats (row_bwd.cu).
cudaError_t launch_param_grad_reduce(const float* part, int nparts, int width, float* out, cudaStream_t s);
// theta[j] = atan2(s_j, c_j) from a.gate (a.width channels).
cudaError_t launch_residual_gate_angles(const ResidualArgs& a, float* theta, cudaStream_t s);

// Returns cudaSuccess or the launch error.
// launch_row: TMA-pipelined kernels (row_tma.cu), falling back to
// launch_row_regs (register-staged, row_norm.cu) for rows too wide to stage.
cudaError_t launch_row(int dtype, RowOp op, const RowArgs& a, cudaStream_t s);
cudaError_t launch_row_regs(int dtype, RowOp op, const RowArgs& a, cudaStream_t s);
// Device-side error words: nonzero once a bounded mbarrier wait of the row
// pipeline (read_device_error) or of the Q/K ring (read_qk_device_error)
// timed out.
cudaError_t read_device_error(unsigned int* out, bool clear);
cudaError_t read_qk_device_error(unsigned int* out, bool clear);
cudaError_t read_bwd_device_error(unsigned int* out, bool clear);
cudaError_t launch_head_gate(int dtype, const HeadGateArgs& a, cudaStream_t s);
cudaError_t launch_qk(int dtype, int use_rope, int upcast_rope, const QkArgs& a, cudaStream_t s);
cudaError_t launch_copy(const void* src, void* dst, int64_t bytes, cudaStream_t s);
// Row backward: per-CTA partials into a.part_gain / a.part_theta (the caller's
// workspace), then a deterministic reduction into dgain / dtheta (either may
// be null).
cudaError_t launch_row_bwd(int dtype, BwdOp op, RowBwdArgs a, float* dgain, float* dtheta,
                           cudaStream_t s);

// Device facts for grid sizing (cached per device).
int sm_count();
int blocks_per_sm(const void* kernel, int threads, size_t dyn_smem = 0);

}  // namespace muse
