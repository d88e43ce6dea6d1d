/*
 * muse_oracle.h - plain, slow, double-precision CPU oracle for the five fused
 * per-token normalisation cores of the Muse Spark Open decoder layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check of the entry
 * module and the benchmark's CPU-baseline leg may load this library.  It
 * shares no code, header, table or constant with the CUDA library.
 *
 * Source of every definition: the NeMo AutoModel API reference page
 * "nemo_automodel.components.models.muse_spark.layers" (versions 0.4 and
 * latest), entries _rms_norm_core, _input_scale_norm_core, _qk_norm_rope_core,
 * _output_norm_gate_core, _norm_residual_core, apply_rotary_embedding,
 * MuseSparkRotaryEmbedding, MuseSparkRMSNorm and MuseSparkResidual.  Where the
 * page leaves a step open the reading is stated beside the function.
 *
 * Conventions
 *   - bf16 tensors are passed as uint16_t bit patterns, f32 tensors as float.
 *   - dtype: 0 = bf16, 1 = f32.
 *   - All tensors are contiguous and row-major.
 *   - Every function writes `out` in the output dtype (what the pages' core
 *     returns) and, when the pointers are not NULL, three double arrays of the
 *     same element count used by parity checks:
 *       lo[i], hi[i]  the smallest and largest exact (real-valued) result
 *                     before the final cast, over every bf16 value that an
 *                     intermediate cast may legitimately take (see below);
 *                     lo == hi when no intermediate cast is in doubt;
 *       mag[i]        the sum of the magnitudes of the terms that form the
 *                     result before its final cast (|y| for a plain product,
 *                     |a*c| + |b*s| for a rotation, |cos*h| + |sin*nb| for the
 *                     residual blend).  A checker scales its FP32 evaluation
 *                     allowance by it.
 *   - Intermediate casts to bf16 (the normalised Q/K cast, the query_scale
 *     cast, the v2 rotation's cos/sin casts, the branch cast before the
 *     residual blend) are taken to round-to-nearest-even.  An FP32
 *     evaluation of the same real value differs from it by far less than
 *     2^-20 relative; when the real value lies within 2^-20 (relative) of a
 *     bf16 rounding midpoint, both neighbouring bf16 values are admissible
 *     results of that cast and the oracle carries both forward.
 *   - Return value: 0 on success, -1 on an invalid argument.
 */
#ifndef MUSE_ORACLE_H
#define MUSE_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Relative distance to a bf16 rounding midpoint below which an intermediate
 * cast is treated as admitting both neighbours. */
#define MUSE_ORACLE_AMBIG_REL 0x1p-20

int muse_oracle_version(void);

/* Round each double to the nearest bfloat16 (ties to even) and return its
 * bit pattern.  NaN maps to a quiet NaN of the same sign. */
void muse_oracle_round_bf16(const double* v, uint16_t* bits, int64_t n);

/* FP32 RoPE inverse frequencies: inv_freq[i] = f32(base^(-2i/head_dim)),
 * i = 0 .. head_dim/2 - 1 (MuseSparkRotaryEmbedding: FP32 frequencies,
 * cos/sin of width head_dim/2). */
int muse_oracle_inv_freq(int32_t head_dim, float base, float* inv_freq);

/* Positions used when the caller passes none.
 *   layout 0 (BSHD): tokens = batch*seqlen, pos[t] = t mod seqlen.
 *   layout 1 (THD):  pos[t] = t - cu_seqlens[d] for the document d whose
 *                    range [cu_seqlens[d], cu_seqlens[d+1]) holds t.
 * cu_seqlens (THD only) has num_seqs+1 entries, starts at 0, does not
 * decrease and ends at total_tokens. */
int muse_oracle_positions(int layout, int64_t batch, int64_t seqlen,
                          const int32_t* cu_seqlens, int32_t num_seqs,
                          int64_t total_tokens, int32_t* pos);

/* Core 1, _rms_norm_core: y = cast((x * r(x)) * w_eff), r(x) = 1/sqrt(mean(x^2)+eps),
 * w_eff[j] = f32(gain[j] + gain_offset); no gain multiply when gain == NULL. */
int muse_oracle_rms_norm(int dtype, const void* x, int64_t rows, int64_t hidden,
                         const float* gain, float gain_offset, float eps,
                         void* out, double* lo, double* hi, double* mag);

/* Per-expert core 1 (MuseSparkMoE pre_expert_norm / post_expert_norm): rows
 * [offsets[g], offsets[g+1]) use gain row g of gains [num_groups, hidden]. */
int muse_oracle_rms_norm_grouped(int dtype, const void* x, int64_t rows, int64_t hidden,
                                 const float* gains, float gain_offset, const int32_t* offsets,
                                 int32_t num_groups, float eps, void* out, double* lo, double* hi,
                                 double* mag);

/* Core 1 with separate input and output dtypes (y = cast_out((x r(x)) w_eff));
 * muse_oracle_rms_norm is the case in_dtype == out_dtype. */
int muse_oracle_rms_norm_to(int in_dtype, int out_dtype, const void* x, int64_t rows,
                            int64_t hidden, const float* gain, float gain_offset, float eps,
                            void* out, double* lo, double* hi, double* mag);

/* Core 2, _input_scale_norm_core: z = x * w_eff, y = cast(z * r(z)). */
int muse_oracle_input_scale_norm(int dtype, const void* x, int64_t rows, int64_t hidden,
                                 const float* gain, float gain_offset, float eps,
                                 void* out, double* lo, double* hi, double* mag);

/* Core 3, _qk_norm_rope_core, on q [tokens, hq, d] and k [tokens, hkv, d]
 * with explicit positions pos[tokens]:
 *   n = cast(x * r(x)) per head over d;
 *   query heads only: n = cast(n * query_scale);
 *   use_rope: pairs (2i, 2i+1), phi = f32(f32(pos) * inv_freq[i]),
 *     FP32 rotation (upcast_rope != 0, or dtype f32):
 *        y0 = a cos(phi) - b sin(phi), y1 = a sin(phi) + b cos(phi), one cast;
 *     bf16 rotation (upcast_rope == 0, dtype bf16):
 *        c = bf16(cos phi), s = bf16(sin phi),
 *        y0 = bf16(bf16(a c) - bf16(b s)), y1 = bf16(bf16(a s) + bf16(b c)).
 * The *_lo/_hi/_mag arrays may be NULL. */
int muse_oracle_qk_norm_rope(int dtype, const void* q, const void* k, int64_t tokens,
                             int32_t hq, int32_t hkv, int32_t head_dim,
                             const int32_t* pos, float eps, float query_scale,
                             int use_rope, int upcast_rope, float rope_base,
                             void* q_out, double* q_lo, double* q_hi, double* q_mag,
                             void* k_out, double* k_lo, double* k_hi, double* k_mag);

/* Core 4, _output_norm_gate_core, on o and g [tokens, heads, head_dim]:
 * y = cast(o * r(o) * sigmoid(g)), r over consecutive groups of norm_group
 * elements (norm_group = head_dim: per head; = heads*head_dim: whole token),
 * sigmoid(g) = 1/(1+exp(-g)). */
int muse_oracle_output_norm_gate(int dtype, const void* o, const void* g, int64_t tokens,
                                 int32_t heads, int32_t head_dim, int32_t norm_group,
                                 float eps, void* out, double* lo, double* hi, double* mag);

/* Core 5, _norm_residual_core with the declared blend:
 *   nb = cast_branch(normed(branch)), normed = core 1 form (input_scale == 0)
 *        or core 2 form (input_scale != 0) with w_eff and norm_eps;
 *   h' = f32(cos(theta) * h + sin(theta) * nb), per channel theta (FP32). */
int muse_oracle_norm_residual(const float* stream, int branch_dtype, const void* branch,
                              int64_t rows, int64_t hidden, const float* gain,
                              float gain_offset, const float* theta, int input_scale,
                              float norm_eps, float* out, double* lo, double* hi,
                              double* mag);

/* _residual_core / MuseSparkResidual without a branch norm, with core 5's
 * declared blend: h' = f32(cos(theta) h + sin(theta) branch), per channel. */
int muse_oracle_residual_blend(const float* stream, int branch_dtype, const void* branch,
                               int64_t rows, int64_t hidden, const float* theta, float* out,
                               double* lo, double* hi, double* mag);

/* The declared reading of the learned gate (gate, temperature, eps):
 * c^2 = max(sigmoid(gate/temperature), eps), s^2 = 1 - c^2, theta = atan2(s, c). */
int muse_oracle_residual_gate_coefficients(const float* gate, int64_t hidden, float temperature,
                                           float eps, double* c, double* s, double* theta);

/* _residual_core(stream, branch, gate, temperature, eps): h' = c h + s branch. */
int muse_oracle_residual(const float* stream, int branch_dtype, const void* branch, int64_t rows,
                         int64_t hidden, const float* gate, float temperature, float eps, float* out,
                         double* lo, double* hi, double* mag);

/* ---------------------------------------------------------------- backward
 *
 * Gradients of the five cores (the cores run under autograd): the derivative
 * of each forward map, where every dtype boundary the forward materialises
 * passes the gradient back rounded to that tensor's dtype (round_grads != 0;
 * 0 gives the exact derivative).  Input gradients in the input dtype with
 * lo/hi/mag as for the forward; parameter gradients (gain, theta) as [lo, hi]
 * of the exact FP32-free row sum and the sum of the magnitudes of its terms.
 * Any check or parameter array may be NULL.
 *
 * Core 1:  g = dy * w_eff;  dx = r g - r^3 x (sum_j g_j x_j) / H;
 *          dgain = sum over rows of dy * x * r.
 * Core 2:  z = x * w_eff;  dz = r dy - r^3 z (sum_j dy_j z_j) / H;
 *          dx = dz * w_eff;  dgain = sum over rows of dz * x. */
int muse_oracle_rms_norm_bwd(int dtype, const void* x, const void* dy, int64_t rows,
                             int64_t hidden, const float* gain, float gain_offset, float eps,
                             void* dx, double* lo, double* hi, double* mag, double* dgain_lo,
                             double* dgain_hi, double* dgain_mag);
int muse_oracle_input_scale_norm_bwd(int dtype, const void* x, const void* dy, int64_t rows,
                                     int64_t hidden, const float* gain, float gain_offset,
                                     float eps, void* dx, double* lo, double* hi, double* mag,
                                     double* dgain_lo, double* dgain_hi, double* dgain_mag);

/* Core 3.  FP32 (legacy) rotation: dm = R(phi)^T dy; dn = cast(dm), query
 * heads dn = cast(dn * query_scale).  v2 rotation (upcast_rope = 0, bf16
 * tensors; C = cast(cos), S = cast(sin)): dn = cast(cast(dy0 C) + cast(dy1 S)),
 * cast(cast(dy1 C) - cast(dy0 S)) per pair, query heads cast(dn * query_scale).
 * Then dx = r dn - r^3 x (sum_j dn_j x_j) / d. */
int muse_oracle_qk_norm_rope_bwd(int dtype, const void* q, const void* k, const void* dq_out,
                                 const void* dk_out, int64_t tokens, int32_t hq, int32_t hkv,
                                 int32_t head_dim, const int32_t* pos, float eps,
                                 float query_scale, int use_rope, int upcast_rope, float rope_base,
                                 int round_grads, void* dq, double* dq_lo, double* dq_hi,
                                 double* dq_mag, void* dk, double* dk_lo, double* dk_hi,
                                 double* dk_mag);

/* Core 4: s = sigmoid(g), n = o r(o); dn = dy s;
 * do = r dn - r^3 o (sum_j dn_j o_j) / G;  dg = dy n s (1 - s). */
int muse_oracle_output_norm_gate_bwd(int dtype, const void* o, const void* g, const void* dy,
                                     int64_t tokens, int32_t heads, int32_t head_dim,
                                     int32_t norm_group, float eps, void* d_o, double* do_lo,
                                     double* do_hi, double* do_mag, void* dg, double* dg_lo,
                                     double* dg_hi, double* dg_mag);

/* Core 5: dh = cos(theta) dh';  dnb = cast_branch(sin(theta) dh');
 * dbranch = core 1 (input_scale == 0) or core 2 backward of dnb;
 * dgain = that backward's gain gradient;
 * dtheta = sum over rows of dh' (-sin(theta) h + cos(theta) nb). */
int muse_oracle_norm_residual_bwd(const float* stream, int branch_dtype, const void* branch,
                                  const float* dstream_out, int64_t rows, int64_t hidden,
                                  const float* gain, float gain_offset, const float* theta,
                                  int input_scale, float norm_eps, int round_grads,
                                  float* dstream, double* ds_lo, double* ds_hi, double* ds_mag,
                                  void* dbranch, double* db_lo, double* db_hi, double* db_mag,
                                  double* dgain_lo, double* dgain_hi, double* dgain_mag,
                                  double* dtheta_lo, double* dtheta_hi, double* dtheta_mag);

/* Backward of _residual_core: dstream = c dy (FP32), dbranch = cast_branch(s dy),
 * and the angle (dtheta) or gate (dgate) gradient as a sum over rows, returned as
 * (lo, hi, mag) double triples. */
int muse_oracle_residual_blend_bwd(const float* stream, int branch_dtype, const void* branch,
                                   const float* dy, int64_t rows, int64_t hidden, const float* theta,
                                   float* dstream, double* ds_lo, double* ds_hi, double* ds_mag,
                                   void* dbranch, double* db_lo, double* db_hi, double* db_mag,
                                   double* dtheta_lo, double* dtheta_hi, double* dtheta_mag);
int muse_oracle_residual_bwd(const float* stream, int branch_dtype, const void* branch,
                             const float* dy, int64_t rows, int64_t hidden, const float* gate,
                             float temperature, float eps, float* dstream, double* ds_lo,
                             double* ds_hi, double* ds_mag, void* dbranch, double* db_lo,
                             double* db_hi, double* db_mag, double* dgate_lo, double* dgate_hi,
                             double* dgate_mag);

/* Vision 2-D RoPE (page "...muse_spark.vision": _rope_frequencies,
 * _apply_vision_rope).  Frequencies of one row-major grid, out
 * [grid_h * grid_w, head_dim / 2, 2] = (cos, sin) per pair: the first
 * head_dim / 4 pairs from the patch row, the rest from the column, with
 * frequencies theta^(-2j/(head_dim/2)) (a reading; the page gives the shape).
 * The rotation: y[2i] = a c - b s, y[2i+1] = a s + b c per token and head
 * with the token's (c, s) from freqs [tokens, head_dim / 2, 2], one cast. */
int muse_oracle_vision_rope_frequencies(int32_t head_dim, int32_t grid_h, int32_t grid_w,
                                        float theta, float* out);
int muse_oracle_vision_rope(int dtype, const void* q, const void* k, int64_t tokens, int32_t hq,
                            int32_t hk, int32_t head_dim, const float* freqs, void* q_out,
                            double* q_lo, double* q_hi, double* q_mag, void* k_out, double* k_lo,
                            double* k_hi, double* k_mag);

#ifdef __cplusplus
}
#endif

#endif /* MUSE_ORACLE_H */
