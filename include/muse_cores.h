/*
 * muse_cores.h - C ABI of the B200 (sm_100a) fused per-token normalisation
 * cores of the Muse Spark Open decoder layer.
 *
 * The five cores restate the pure functions documented on the NeMo AutoModel
 * API reference page "nemo_automodel.components.models.muse_spark.layers":
 * _rms_norm_core, _input_scale_norm_core, _qk_norm_rope_core,
 * _output_norm_gate_core and _norm_residual_core.  Each entry point launches
 * one CUDA kernel that makes one pass over HBM.
 *
 * Common contract
 *   - Every pointer to tensor data is a DEVICE pointer owned by the caller;
 *     the library allocates no memory and keeps no per-call state.  The
 *     only process-wide state is a cache of SM counts and occupancy figures.
 *   - Every call is asynchronous on `stream` (NULL = the legacy default
 *     stream of the current device) and never synchronises.  Results are
 *     valid once work queued on `stream` after the call has completed.
 *   - Tensors are row-major.  A "row stride" counts ELEMENTS between the
 *     first elements of consecutive rows (tokens) and must be >= the row width.
 *   - dtype is the activation dtype; every output keeps the dtype of the
 *     tensor it replaces (the residual stream stays FP32).  Gains
 *     and blend angles are FP32; every reduction and every product runs in
 *     FP32.
 *   - Aliasing: an output may be the very same memory as its input (same
 *     pointer, same stride: in-place); any other overlap between an output and
 *     any tensor of the call returns MUSE_ERR_INVALID_ARGUMENT.
 *   - rows/tokens == 0 returns MUSE_OK without a launch.
 *   - Limits (MUSE_ERR_UNSUPPORTED): every tensor pointer (gains and blend
 *     angles included) and every row stride in bytes must be a multiple of
 *     16 bytes, and every row width (and head_dim) a multiple of 8 elements
 *     for bf16 or 4 for f32 (16 bytes).  positions and cu_seqlens need 4-byte
 *     alignment.  Row widths up to MUSE_MAX_ROW_BYTES bytes; head_dim up to
 *     512 bytes (256 bf16 or 128 f32 elements).
 *   - Errors: a status is returned before anything is launched when an
 *     argument is invalid; MUSE_ERR_CUDA reports a failed launch (the CUDA
 *     error is cleared).  muse_last_error() gives a one-line description of
 *     the last failing call on the calling thread.
 */
#ifndef MUSE_CORES_H
#define MUSE_CORES_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MUSE_VERSION 1
/* Widest row a single CTA normalises: 32768 bf16 or 16384 f32 elements. */
#define MUSE_MAX_ROW_BYTES 65536

typedef enum muse_status {
    MUSE_OK = 0,
    MUSE_ERR_INVALID_ARGUMENT = 1,
    MUSE_ERR_UNSUPPORTED = 2,
    MUSE_ERR_CUDA = 3
} muse_status;

typedef enum muse_dtype { MUSE_DTYPE_BF16 = 0, MUSE_DTYPE_F32 = 1 } muse_dtype;

typedef enum muse_layout { MUSE_LAYOUT_BSHD = 0, MUSE_LAYOUT_THD = 1 } muse_layout;

int muse_version(void);
const char* muse_status_string(muse_status s);
/* Description of the last non-OK status returned on this thread ("" if none). */
const char* muse_last_error(void);

/*
 * Core 1 - _rms_norm_core (FP32 normalisation, then the effective gain, then
 * the single cast to the output dtype; MuseSparkRMSNorm, zero-centered gain).
 *   y[r, j] = cast( (x[r, j] * inv_rms(x[r, :])) * w_eff[j] ),
 *   inv_rms(v) = 1 / sqrt(mean_j(v_j^2) + eps),
 *   w_eff[j] = f32(gain[j] + gain_offset)   (gain_offset 1.0 for the
 *   zero-centered checkpoint gain, 0 otherwise); gain == NULL: no multiply.
 * x [rows, hidden] with row stride x_row_stride, y [rows, hidden] with row
 * stride y_row_stride, both `dtype`; gain [hidden] FP32 or NULL.
 */
muse_status muse_rms_norm(const void* x, void* y, muse_dtype dtype, int64_t rows,
                          int64_t hidden, int64_t x_row_stride, int64_t y_row_stride,
                          const float* gain, float gain_offset, float eps,
                          cudaStream_t stream);

/*
 * Core 2 - _input_scale_norm_core (the effective gain scales the row first;
 * the FP32 norm and its eps then act on the SCALED activation).
 *   z[r, j] = x[r, j] * w_eff[j]  (FP32),  y[r, j] = cast( z[r, j] * inv_rms(z[r, :]) ).
 * Arguments as muse_rms_norm.
 */
muse_status muse_input_scale_norm(const void* x, void* y, muse_dtype dtype, int64_t rows,
                                  int64_t hidden, int64_t x_row_stride, int64_t y_row_stride,
                                  const float* gain, float gain_offset, float eps,
                                  cudaStream_t stream);

/*
 * Core 3 - _qk_norm_rope_core (per-head Q/K normalisation and rotation that
 * keeps every cast of the checkpoint in place), with the rotary frequencies of
 * MuseSparkRotaryEmbedding and the adjacent-pair rotation of
 * apply_rotary_embedding computed in the kernel from positions.
 * Per token t and per head (hq query heads, hkv key heads), over head_dim D:
 *   n = cast( x * inv_rms(x) );  query heads only: n = cast( n * query_scale );
 *   use_rope: for pair i = 0 .. D/2-1 with (a, b) = (n[2i], n[2i+1]),
 *     phi = f32( f32(pos_t) * inv_freq[i] ),  inv_freq[i] = f32(rope_base^(-2i/D));
 *     upcast_rope != 0 (original checkpoint, FP32 rotation):
 *       y[2i] = cast(a cos(phi) - b sin(phi)), y[2i+1] = cast(a sin(phi) + b cos(phi));
 *     upcast_rope == 0 (HF release, rotation in the Q/K dtype):
 *       c = cast(cos phi), s = cast(sin phi),
 *       y[2i] = cast(cast(a c) - cast(b s)), y[2i+1] = cast(cast(a s) + cast(b c)).
 * q [T, hq, D] with token stride q_tok_stride, k [T, hkv, D] with
 * k_tok_stride (views into a fused QKV projection are fine); outputs with
 * their own token strides; heads of one token are contiguous.
 * Tokens: BSHD: T = batch * seqlen; THD: T = total_tokens.
 * positions: int32 [T] device array, or NULL to derive them:
 *   BSHD: pos_t = t mod seqlen;  THD: pos_t = t - cu_seqlens[d] for the
 *   document d with cu_seqlens[d] <= t < cu_seqlens[d+1].
 * cu_seqlens: int32 [num_seqs+1] device array (THD with positions == NULL
 * only; otherwise ignored).  It must start at 0, not decrease and end at
 * total_tokens; the library cannot check device contents without a
 * synchronisation, so other contents give unspecified positions (never an
 * out-of-bounds access).  Under context parallelism pass positions.
 * Requires hq % hkv == 0 (GQA), D even, D <= 256.
 */
muse_status muse_qk_norm_rope(const void* q, const void* k, void* q_out, void* k_out,
                              muse_dtype dtype, muse_layout layout, int64_t batch,
                              int64_t seqlen, const int32_t* cu_seqlens, int32_t num_seqs,
                              int64_t total_tokens, const int32_t* positions, int32_t hq,
                              int32_t hkv, int32_t head_dim, int64_t q_tok_stride,
                              int64_t k_tok_stride, int64_t q_out_tok_stride,
                              int64_t k_out_tok_stride, float eps, float query_scale,
                              int use_rope, int upcast_rope, float rope_base,
                              cudaStream_t stream);

/*
 * Core 4 - _output_norm_gate_core (norm without gain of the attention output,
 * times the sigmoid of the gate projection; both in FP32, one cast).
 *   y = cast( o * inv_rms(o over its group) * sigmoid(g) ),  sigmoid(g) = 1/(1+exp(-g)).
 * o, gate, y: [tokens, heads, head_dim] contiguous, `dtype`.
 * norm_group = head_dim: one norm per head (the head-split layout the page
 * passes); norm_group = heads*head_dim: one norm per token.
 */
muse_status muse_output_norm_gate(const void* o, const void* gate, void* y, muse_dtype dtype,
                                  int64_t tokens, int32_t heads, int32_t head_dim,
                                  int32_t norm_group, float eps, cudaStream_t stream);

/*
 * Core 5 - _norm_residual_core (branch norm, cast back to the branch dtype,
 * then blended into the FP32 stream) with the learned blend of
 * MuseSparkResidual read as a per-channel rotation by theta:
 *   nb[r, j] = cast_branch( normed(branch[r, :])[j] ),  normed = core 1's form
 *     (input_scale == 0: gain after the norm) or core 2's form (input_scale != 0),
 *     with w_eff = f32(gain + gain_offset) (gain may be NULL) and norm_eps;
 *   stream_out[r, j] = cos(theta[j]) * stream_in[r, j] + sin(theta[j]) * nb[r, j]   (FP32).
 * stream_in, stream_out: FP32 [rows, hidden] contiguous (stream_out ==
 * stream_in is allowed); branch: [rows, hidden] contiguous, branch_dtype;
 * gain, theta: FP32 [hidden].
 */
muse_status muse_norm_residual(const float* stream_in, const void* branch, float* stream_out,
                               muse_dtype branch_dtype, int64_t rows, int64_t hidden,
                               const float* gain, float gain_offset, const float* theta,
                               int input_scale, float norm_eps, cudaStream_t stream);

/*
 * _residual_core / MuseSparkResidual.forward (layers page: "blend the
 * residual and branch using the checkpoint's learned gate"; a learned
 * norm-preserving residual connection) - the blend without a branch norm.
 * The page gives no formula; two forms are offered:
 *
 * muse_residual_blend - the blend core 5 uses, per channel j:
 *   stream_out[r, j] = cos(theta[j]) * stream_in[r, j] + sin(theta[j]) * f32(branch[r, j])
 *   (FP32 arithmetic; the branch is read as it is, no cast).
 * muse_residual - the page's signature (gate, temperature, eps), read as
 *   c^2 = max(sigmoid(gate[j] / temperature), eps)   (eps: the lower bound on
 *         the squared residual coefficient),  s^2 = 1 - c^2,  c, s >= 0,
 *   stream_out[r, j] = c * stream_in[r, j] + s * f32(branch[r, j]),
 *   i.e. muse_residual_blend with theta = atan2(s, c).  temperature finite
 *   and > 0, eps in [0, 1], else MUSE_ERR_INVALID_ARGUMENT.  The page's
 *   defaults are temperature 0.3 and eps 0.001.
 * stream_in, stream_out: FP32 [rows, hidden] contiguous (stream_out ==
 * stream_in is allowed); branch: [rows, hidden] contiguous in branch_dtype;
 * theta / gate: FP32 [hidden].  Pointers 16-byte aligned and hidden a
 * multiple of 16 bytes of the branch dtype, else MUSE_ERR_UNSUPPORTED.
 */
muse_status muse_residual_blend(const float* stream_in, const void* branch, float* stream_out,
                                muse_dtype branch_dtype, int64_t rows, int64_t hidden, const float* theta,
                                cudaStream_t stream);
muse_status muse_residual(const float* stream_in, const void* branch, float* stream_out, muse_dtype branch_dtype,
                          int64_t rows, int64_t hidden, const float* gate, float temperature, float eps,
                          cudaStream_t stream);

/*
 * Backward of _residual_core (both forms), in the convention of the other
 * backward calls (the gradient of every cast the forward materialises is the
 * incoming gradient rounded to that tensor's dtype).  Given the forward's
 * stream_in, branch and theta or gate, and dstream_out = dL/dstream_out (FP32):
 *   dstream_in = c * dstream_out                              (FP32);
 *   dbranch    = cast_branch(s * dstream_out);
 *   dtheta[j]  = sum over rows of dstream_out (c b - s h)     (angle form),
 *   dgate[j]   = sum over rows of dstream_out (dc/dgate h + ds/dgate b)
 *              = c s / (2 temperature) * sum of dstream_out (s h - c b)
 *                where sigmoid(gate / temperature) >= eps, else 0 (gate form).
 * dtheta / dgate may be NULL (then the workspace may be NULL too); otherwise a
 * caller-owned device workspace of muse_residual_backward_workspace_bytes(rows,
 * hidden) bytes (16-byte aligned; contents ignored on entry, undefined on
 * return) holds one partial row per row block, summed in a fixed order.
 * dstream_in may be the very memory of dstream_out, dbranch of branch; nothing
 * else may overlap.  Limits and errors as muse_residual; rows == 0 zeroes
 * dtheta / dgate.
 */
size_t muse_residual_backward_workspace_bytes(int64_t rows, int64_t hidden);
muse_status muse_residual_blend_backward(const float* stream_in, const void* branch, const float* dstream_out,
                                         float* dstream_in, void* dbranch, muse_dtype branch_dtype, int64_t rows,
                                         int64_t hidden, const float* theta, float* dtheta, void* workspace,
                                         size_t workspace_bytes, cudaStream_t stream);
muse_status muse_residual_backward(const float* stream_in, const void* branch, const float* dstream_out,
                                   float* dstream_in, void* dbranch, muse_dtype branch_dtype, int64_t rows,
                                   int64_t hidden, const float* gate, float temperature, float eps, float* dgate,
                                   void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * _residual_core (angle form) fused with the next sublayer's pre-norm, as
 * muse_norm_residual_rms_norm is for core 5: in one pass,
 *   stream_out = muse_residual_blend(stream_in, branch, theta)  (the same values),
 *   y = cast_y((stream_out r(stream_out)) w2),  w2 = next_gain + next_gain_offset
 *       (no multiply when next_gain is NULL), r with next_eps, FP32 arithmetic on
 *       the FP32 values written to stream_out,
 * so the new stream is not read back.  y [rows, hidden] contiguous, FP32 or
 * the branch dtype; y may be the very memory of branch when the dtypes match;
 * stream_out may be stream_in.  Rows up to 1024 16-byte branch vectors, else
 * MUSE_ERR_UNSUPPORTED.  A gate-form caller converts its gate with
 * muse_residual_gate_angles first.
 */
muse_status muse_residual_blend_rms_norm(const float* stream_in, const void* branch, float* stream_out, void* y,
                                         muse_dtype branch_dtype, muse_dtype y_dtype, int64_t rows, int64_t hidden,
                                         const float* theta, const float* next_gain, float next_gain_offset,
                                         float next_eps, cudaStream_t stream);

/*
 * The blend angle of each channel from the learned gate under the reading of
 * muse_residual: theta[j] = atan2(s_j, c_j) in [0, pi/2].  It turns the
 * page's (gate, temperature, residual_eps) of _norm_residual_core into the
 * theta argument of muse_norm_residual / muse_norm_residual_rms_norm.
 * gate, theta: FP32 [hidden], 4-byte aligned; theta may be the very memory
 * of gate; temperature and eps as muse_residual.
 */
muse_status muse_residual_gate_angles(const float* gate, float* theta, int64_t hidden, float temperature,
                                      float eps, cudaStream_t stream);

/*
 * Per-expert form of core 1 (MuseSparkMoE pre_expert_norm / post_expert_norm:
 * per-expert norms over the tokens routed to each expert).  The rows arrive
 * grouped by expert, as a grouped-GEMM dispatch lays them out: rows
 * [group_offsets[g], group_offsets[g+1]) are normalised like
 * muse_rms_norm with the gain row g of gains [num_groups, hidden] (FP32,
 * contiguous) plus gain_offset.  group_offsets is a DEVICE int32 array of
 * num_groups + 1 entries starting at 0, non-decreasing, ending at rows; the
 * library does not read it on the host (a row outside the table uses the
 * nearest group, no access leaves the table).  Rows up to 1024 16-byte
 * vectors, else MUSE_ERR_UNSUPPORTED.
 */
muse_status muse_rms_norm_grouped(const void* x, void* y, muse_dtype dtype, int64_t rows, int64_t hidden,
                                  int64_t x_row_stride, int64_t y_row_stride, const float* gains,
                                  float gain_offset, const int32_t* group_offsets, int32_t num_groups,
                                  float eps, cudaStream_t stream);

/*
 * Vision 2-D RoPE (page "nemo_automodel.components.models.muse_spark.vision":
 * _apply_vision_rope, the adjacent-pair rotation of the NaViT tower's Q/K).
 * Per token t, head and pair i, with (c, s) = freqs[t, i, 0..1]:
 *   y[2i] = a c - b s,   y[2i+1] = a s + b c   (FP32, cast once to dtype),
 * (a, b) = x[2i], x[2i+1].  q [tokens, hq, head_dim], k [tokens, hk,
 * head_dim] (heads contiguous, per-token strides in elements, as the Q/K
 * core), freqs FP32 [tokens, head_dim/2, 2] contiguous (the (cos, sin) of each
 * pair's angle, e.g. from muse_vision_rope_frequencies per grid, concatenated
 * in the packed patch order).  q_out may be the very memory of q, k_out of k;
 * any other overlap is MUSE_ERR_INVALID_ARGUMENT.  Pointers, head rows and
 * strides 16-byte multiples, heads of at most 512 bytes (256 bf16 or 128 f32
 * elements), else MUSE_ERR_UNSUPPORTED.
 */
muse_status muse_vision_rope(const void* q, const void* k, void* q_out, void* k_out, muse_dtype dtype,
                             int64_t tokens, int32_t hq, int32_t hk, int32_t head_dim,
                             int64_t q_tok_stride, int64_t k_tok_stride, int64_t q_out_tok_stride,
                             int64_t k_out_tok_stride, const float* freqs, cudaStream_t stream);

/*
 * The vision RoPE table of one row-major grid_h x grid_w patch grid
 * (_rope_frequencies): out [grid_h * grid_w, head_dim/2, 2] FP32, the (cos,
 * sin) of each pair's angle.  The page gives the shape only; the reading
 * here: pairs i < head_dim/4 take the patch row h, the others the column w,
 * angle = f32(coord) * f32(theta^(-2j/(head_dim/2))), j the pair's index
 * within its half.  head_dim a positive multiple of 4 (at most 512), theta
 * > 0; out 8-byte aligned.
 */
muse_status muse_vision_rope_frequencies(float* out, int32_t head_dim, int32_t grid_h, int32_t grid_w,
                                         float theta, cudaStream_t stream);

/*
 * Core 5 fused with the next sublayer's pre-norm.  The decoder layer updates
 * the FP32 stream with core 5 and then normalises that stream for the next
 * sublayer (MuseSparkDecoderLayer: add_attn, then pre_ffn_norm; add_ffn, then
 * the next layer's input norm).  This call does both in one pass, so the new
 * stream is not read back:
 *   stream_out = core 5 (as muse_norm_residual);
 *   y = cast_y((stream_out r(stream_out)) w2),  w2 = next_gain + next_gain_offset
 *       (no multiply when next_gain is NULL), r with next_eps, FP32 arithmetic
 *       on the FP32 values written to stream_out;
 * y [rows, hidden] contiguous in y_dtype: FP32, or the branch (activation)
 * dtype for a projection input; any other y_dtype is MUSE_ERR_UNSUPPORTED.  y may be the very memory of branch when the dtypes
 * match; stream_out may be stream_in.  Rows up to 1024 16-byte branch vectors
 * (8192 bf16 / 4096 f32 elements), else MUSE_ERR_UNSUPPORTED.
 */
muse_status muse_norm_residual_rms_norm(const float* stream_in, const void* branch, float* stream_out,
                                        void* y, muse_dtype branch_dtype, muse_dtype y_dtype,
                                        int64_t rows, int64_t hidden, const float* gain,
                                        float gain_offset, const float* theta, int input_scale,
                                        float norm_eps, const float* next_gain,
                                        float next_gain_offset, float next_eps,
                                        cudaStream_t stream);

/* ------------------------------------------------------------------ backward
 *
 * The cores run under autograd: the layers page keeps them outside
 * activation-checkpoint caching while "autograd and the enclosing activation
 * checkpoint still run" (_checkpoint_recomputed_math).  The backward calls
 * below compute the derivative of each forward map from the saved forward
 * inputs (r is recomputed), in FP32, where every dtype boundary the forward
 * materialises passes the gradient back rounded to that tensor's dtype, as
 * autograd does through a cast.  Input gradients keep the input dtype;
 * parameter gradients (gain, theta) are FP32 sums over all rows, reduced in a
 * fixed order (bit-reproducible on a given GPU model).
 *
 * Parameter gradients need a caller-owned device workspace of
 * muse_norm_backward_workspace_bytes(rows, hidden) bytes (16-byte aligned;
 * it holds one partial row per CTA; contents on entry are ignored, on return
 * undefined).  Pass dgain / dtheta = NULL to skip a parameter gradient; the
 * workspace may then be NULL too.  Backward rows are limited to 1024 16-byte
 * vectors (8192 bf16 or 4096 f32 elements); wider rows return
 * MUSE_ERR_UNSUPPORTED.  Aliasing: dx may be the very same memory as x or dy
 * (dstream_in as dstream_out, dbranch as branch); dgain, dtheta and the
 * workspace must not overlap anything.  With rows == 0, dgain / dtheta are
 * set to zero.
 */

/* Workspace bytes the row backward calls need for `rows` rows of `hidden`
 * elements on the current device (0 for invalid sizes). */
size_t muse_norm_backward_workspace_bytes(int64_t rows, int64_t hidden);

/*
 * Backward of core 1 (_rms_norm_core).  With w = gain + gain_offset (or 1),
 * r = 1/sqrt(mean(x^2) + eps):
 *   g = dy * w;  dx = r g - r^3 x (sum_j g_j x_j) / hidden;
 *   dgain[j] = sum over rows of dy[j] x[j] r   (when dgain != NULL).
 * x, dy, dx [rows, hidden] in dtype with their own row strides (elements).
 */
muse_status muse_rms_norm_backward(const void* x, const void* dy, void* dx, muse_dtype dtype,
                                   int64_t rows, int64_t hidden, int64_t x_row_stride,
                                   int64_t dy_row_stride, int64_t dx_row_stride,
                                   const float* gain, float gain_offset, float eps, float* dgain,
                                   void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Allocation-free variant of muse_rms_norm_backward (an addition of this
 * library; the API reference pages have no counterpart).  Same arguments and
 * results, without the workspace: the gain partials (one row of `hidden` FP32
 * values per CTA) go to a fixed 16 MiB device array of the library, whose
 * address is looked up once per device on the first call that needs it.
 *   - Allocates nothing and never calls cudaMalloc / cudaFree.
 *   - Every argument is checked first; then a call whose partials exceed the
 *     fixed array is rejected with MUSE_ERR_UNSUPPORTED.  The partials take
 *     one row of hidden floats per CTA of the grid this launch uses
 *     (resident CTAs x SMs, at most 4 per SM, at most one per row): on a
 *     148-SM B200, hidden = 4096 fits at any row count.
 *   - The array is shared by every call on a device: two calls with dgain
 *     must not run concurrently (issue them on one stream, or order their
 *     streams); calls without dgain do not touch it.
 *   - The first call with dgain on each device performs the address lookup,
 *     which must not happen inside a stream capture: make that first call
 *     outside any capture.
 *   - The looked-up address is kept for the life of the process: do not use
 *     this entry point after cudaDeviceReset on that device (the array's
 *     address may change with the new context).
 */
muse_status muse_rms_norm_backward_noalloc(const void* x, const void* dy, void* dx, muse_dtype dtype,
                                           int64_t rows, int64_t hidden, int64_t x_row_stride,
                                           int64_t dy_row_stride, int64_t dx_row_stride,
                                           const float* gain, float gain_offset, float eps,
                                           float* dgain, cudaStream_t stream);

/*
 * Backward of core 2 (_input_scale_norm_core).  z = x w, r = r(z):
 *   dz = r dy - r^3 z (sum_j dy_j z_j) / hidden;  dx = dz w;
 *   dgain[j] = sum over rows of dz[j] x[j].
 */
muse_status muse_input_scale_norm_backward(const void* x, const void* dy, void* dx,
                                           muse_dtype dtype, int64_t rows, int64_t hidden,
                                           int64_t x_row_stride, int64_t dy_row_stride,
                                           int64_t dx_row_stride, const float* gain,
                                           float gain_offset, float eps, float* dgain,
                                           void* workspace, size_t workspace_bytes,
                                           cudaStream_t stream);

/*
 * Backward of core 5 (_norm_residual_core, blend h' = cos(theta) h +
 * sin(theta) nb).  Given the forward's stream_in h, branch and theta, and
 * dstream_out = dL/dh':
 *   dstream_in = cos(theta) dstream_out                       (FP32);
 *   dnb = cast_branch(sin(theta) dstream_out);
 *   dbranch = the core 1 (input_scale == 0) or core 2 backward of dnb;
 *   dgain = that backward's gain gradient;
 *   dtheta[j] = sum over rows of dstream_out (-sin(theta) h + cos(theta) nb),
 *     nb the forward's cast normalised branch.
 * All rows contiguous [rows, hidden].
 */
muse_status muse_norm_residual_backward(const float* stream_in, const void* branch,
                                        const float* dstream_out, float* dstream_in,
                                        void* dbranch, muse_dtype branch_dtype, int64_t rows,
                                        int64_t hidden, const float* gain, float gain_offset,
                                        const float* theta, int input_scale, float norm_eps,
                                        float* dgain, float* dtheta, void* workspace,
                                        size_t workspace_bytes, cudaStream_t stream);

/*
 * Backward of core 4 (_output_norm_gate_core).  Per norm group of G
 * elements (norm_group = head_dim or heads*head_dim, as in the forward):
 *   s = sigmoid(gate), n = o r(o), dn = dy s;
 *   d_o = r dn - r^3 o (sum_j dn_j o_j) / G;   dgate = dy n s (1 - s).
 * o, gate, dy, d_o, dgate contiguous [tokens, heads, head_dim] in dtype.
 * d_o may be the very memory of o or dy, dgate of gate or dy.
 */
muse_status muse_output_norm_gate_backward(const void* o, const void* gate, const void* dy, void* d_o,
                                           void* dgate, muse_dtype dtype, int64_t tokens,
                                           int32_t heads, int32_t head_dim, int32_t norm_group,
                                           float eps, cudaStream_t stream);

/*
 * Backward of core 3 (_qk_norm_rope_core; the rotation modes of
 * MuseSparkAttention's upcast_rope and apply_rotary_embedding).  Per token
 * and head, with phi the forward's FP32 angle (same positions rule and
 * layouts as muse_qk_norm_rope):
 *   upcast_rope != 0 (legacy, FP32 rotation), or FP32 tensors:
 *     dm = R(phi)^T dy, i.e. per pair (c dy0 + s dy1, -s dy0 + c dy1), FP32;
 *     dn = cast(dm);
 *   upcast_rope == 0 on bf16 (v2: the forward's products and sums in bf16,
 *   C, S = bf16 cos and sin of phi), the gradient through those operations:
 *     dn = (cast(cast(dy0 C) + cast(dy1 S)), cast(cast(dy1 C) - cast(dy0 S)));
 *   query heads: dn = cast(dn * query_scale);
 *   dx = r dn - r^3 x (sum_j dn_j x_j) / head_dim, cast to dtype.
 * q, k are the forward's inputs; dq_out, dk_out the incoming gradients; dq,
 * dk the results, each with its own token stride (elements).  dq may be the
 * very memory of q or dq_out, dk of k or dk_out.
 */
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
                                       cudaStream_t stream);

/*
 * Device-side error flags of the current device, for diagnostics.  The row
 * kernels (cores 1, 2, 5, core 4 per token), the Q/K kernel (core 3) and the
 * row and Q/K backward kernels stream their inputs through shared memory with bulk
 * copies tracked by mbarriers; every wait on one is bounded, and a wait that
 * gives up sets bit 0 (row kernels), bit 1 (Q/K kernel), bit 2 (row
 * backward) or bit 3 (Q/K backward) of the flags (and the affected warps
 * stop writing).  *flags receives them; clear != 0 resets them.  Synchronous: it
 * waits for the device.  Returns MUSE_ERR_INVALID_ARGUMENT for a NULL flags
 * pointer, MUSE_ERR_CUDA if the copy fails.
 */
muse_status muse_device_error(unsigned int* flags, int clear);

/*
 * Bounded-wait probe (diagnostics; an addition of this library, the API
 * reference pages have no counterpart).  It runs muse_rms_norm's kernel with
 * one planted wait that cannot complete, so that a test can drive the
 * failure handling of the bulk-copy pipeline without faulting or hanging the
 * GPU.  Arguments as muse_rms_norm, plus:
 *   spin_limit: polls per mbarrier wait before it gives up, 1 .. 2^24 (the
 *     ordinary calls use 2^24);
 *   stall_row: a row in [0, rows).  The producer warp of the CTA that owns
 *     this row never signals the row's pipeline stage and issues no copy for
 *     it or for that CTA's later rows.
 * Expected outcome: every other CTA's rows are normalised as by
 * muse_rms_norm; in the stalled CTA, the rows before stall_row are too, the
 * consumer warps give up on stall_row after spin_limit polls, set bit 0 of
 * muse_device_error, and write nothing from stall_row on; the producer waits
 * (bounded) for the copies it did issue before the CTA exits, so no copy is
 * left in flight.  Rows must be at most 16384 bytes (else
 * MUSE_ERR_UNSUPPORTED); spin_limit or stall_row out of range is
 * MUSE_ERR_INVALID_ARGUMENT.  Not for production use.
 */
muse_status muse_rms_norm_stall_probe(const void* x, void* y, muse_dtype dtype, int64_t rows,
                                      int64_t hidden, int64_t x_row_stride, int64_t y_row_stride,
                                      const float* gain, float gain_offset, float eps,
                                      uint32_t spin_limit, int64_t stall_row, cudaStream_t stream);

/*
 * Bandwidth reference (not a core): copy `bytes` bytes from src to dst with
 * 16-byte vector loads and stores over a persistent grid.  It measures the
 * HBM roofline on the same device the cores run on.  bytes % 16 == 0; both
 * pointers 16-byte aligned; the ranges must not overlap.
 */
muse_status muse_stream_copy(const void* src, void* dst, int64_t bytes, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MUSE_CORES_H */
