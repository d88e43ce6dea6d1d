/*
 * muse_oracle.c - plain double-precision CPU oracle for the five Muse Spark
 * Open normalisation cores.  TEST INFRASTRUCTURE ONLY (see muse_oracle.h):
 * only tests, the entry module's smoke check and the benchmark's CPU-baseline
 * leg load it; the CUDA library never does.
 *
 * Every function is the definition written out: loops over rows, heads and
 * pairs; sums of squares, products, square roots, sines, cosines and
 * exponentials in double; rounding to bf16 or FP32 exactly where the API
 * reference page "nemo_automodel.components.models.muse_spark.layers" puts a
 * dtype boundary.  No blocking, fusion or reordering.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared (no -ffast-math: every rounding here
 * is IEEE round-to-nearest-even).
 */
#include "muse_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define DT_BF16 0
#define DT_F32 1

int muse_oracle_version(void) { return 1; }

/* ---------------------------------------------------------------- rounding */

/* Nearest bfloat16 value to v, ties to even, returned as a double (every
 * bfloat16 value is exactly representable in double).  bfloat16 keeps 8
 * significant bits for normal numbers (exponent >= -126) and a fixed spacing
 * of 2^-133 below that; the largest finite value is (2 - 2^-7) * 2^127. */
static double bf16_round(double v) {
    if (isnan(v) || isinf(v) || v == 0.0) return v;
    double a = fabs(v);
    int e;
    frexp(a, &e);              /* a in [2^(e-1), 2^e) */
    int q = e - 8;             /* spacing of 8 significant bits */
    if (q < -133) q = -133;    /* subnormal spacing */
    double s = ldexp(a, -q);   /* exact scaling */
    double r = nearbyint(s);   /* default rounding mode: ties to even */
    double res = ldexp(r, q);
    if (res >= 0x1p128) res = INFINITY;
    return copysign(res, v);
}

static uint16_t bf16_bits(double rounded) {
    if (isnan(rounded)) return signbit(rounded) ? 0xFFC0u : 0x7FC0u;
    float f = (float)rounded; /* exact: rounded is a bfloat16 value */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

static double bf16_value(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round to the tensor dtype. */
static double cast_to(int dtype, double v) {
    return dtype == DT_BF16 ? bf16_round(v) : (double)(float)v;
}

static double load_elem(int dtype, const void* p, int64_t i) {
    return dtype == DT_BF16 ? bf16_value(((const uint16_t*)p)[i])
                            : (double)((const float*)p)[i];
}

/* Store v (not yet rounded) in the tensor dtype. */
static void store_elem(int dtype, void* p, int64_t i, double v) {
    if (dtype == DT_BF16)
        ((uint16_t*)p)[i] = bf16_bits(bf16_round(v));
    else
        ((float*)p)[i] = (float)v;
}

/* The values an intermediate cast of the real value v may take.  c[0] is the
 * round-to-nearest-even result.  For bf16, when v lies within
 * MUSE_ORACLE_AMBIG_REL * |v| of a rounding midpoint, the other neighbour is
 * returned as c[1] too (an FP32 evaluation of v can land on either side).
 * FP32 casts keep one value; their evaluation error is continuous and is
 * covered by the checker's allowance. */
static int cast_candidates(int dtype, double v, double c[2]) {
    c[0] = cast_to(dtype, v);
    if (dtype != DT_BF16) return 1;
    double d = fabs(v) * MUSE_ORACLE_AMBIG_REL;
    double lo = bf16_round(v - d), hi = bf16_round(v + d);
    if (lo == hi) return 1;
    c[1] = (lo == c[0]) ? hi : lo;
    return 2;
}

void muse_oracle_round_bf16(const double* v, uint16_t* bits, int64_t n) {
    for (int64_t i = 0; i < n; ++i) bits[i] = bf16_bits(bf16_round(v[i]));
}

/* ------------------------------------------------------------------- RoPE */

int muse_oracle_inv_freq(int32_t head_dim, float base, float* inv_freq) {
    if (head_dim <= 0 || (head_dim & 1) || !(base > 0.0f) || !inv_freq) return -1;
    for (int32_t i = 0; i < head_dim / 2; ++i)
        inv_freq[i] = (float)pow((double)base, -(2.0 * (double)i) / (double)head_dim);
    return 0;
}

int muse_oracle_positions(int layout, int64_t batch, int64_t seqlen,
                          const int32_t* cu_seqlens, int32_t num_seqs,
                          int64_t total_tokens, int32_t* pos) {
    if (!pos) return -1;
    if (layout == 0) {
        if (batch < 0 || seqlen <= 0) return -1;
        for (int64_t t = 0; t < batch * seqlen; ++t) pos[t] = (int32_t)(t % seqlen);
        return 0;
    }
    if (layout != 1 || !cu_seqlens || num_seqs < 0) return -1;
    if (cu_seqlens[0] != 0 || cu_seqlens[num_seqs] != total_tokens) return -1;
    for (int32_t d = 0; d < num_seqs; ++d) {
        if (cu_seqlens[d + 1] < cu_seqlens[d]) return -1;
        for (int64_t t = cu_seqlens[d]; t < cu_seqlens[d + 1]; ++t)
            pos[t] = (int32_t)(t - cu_seqlens[d]);
    }
    return 0;
}

/* ------------------------------------------------------------ shared bits */

/* r(x) = 1 / sqrt(mean of squares + eps): eps sits inside the square root,
 * added to the mean square (parameter eps of _rms_norm_core). */
static double inv_rms(double sum_sq, int64_t width, float eps) {
    return 1.0 / sqrt(sum_sq / (double)width + (double)eps);
}

/* Effective gain: the zero-centered checkpoint gain plus its offset, summed in
 * FP32 (MuseSparkRMSNorm: gain_center, effective_weight returns the actual
 * multiplicative gain). */
static double eff_gain(const float* gain, float offset, int64_t j) {
    if (!gain) return 1.0;
    float w = gain[j] + offset; /* FP32 addition */
    return (double)w;
}

static void put_check(double* lo, double* hi, double* mag, int64_t i,
                      double l, double h, double m) {
    if (lo) lo[i] = l;
    if (hi) hi[i] = h;
    if (mag) mag[i] = m;
}

static int valid_dtype(int dt) { return dt == DT_BF16 || dt == DT_F32; }

/* ------------------------------------------------------------------ core 1 */

/* _rms_norm_core: normalise in FP32, then apply the effective gain before the
 * one output cast; the output keeps the input dtype. */
int muse_oracle_rms_norm(int dtype, const void* x, int64_t rows, int64_t hidden,
                         const float* gain, float gain_offset, float eps,
                         void* out, double* lo, double* hi, double* mag) {
    return muse_oracle_rms_norm_to(dtype, dtype, x, rows, hidden, gain, gain_offset, eps, out, lo,
                                   hi, mag);
}

/* Core 1 with the output cast to out_dtype (the pre-norm of the FP32 stream
 * feeding a projection may be asked for in the activation dtype). */
int muse_oracle_rms_norm_to(int in_dtype, int out_dtype, const void* x, int64_t rows,
                            int64_t hidden, const float* gain, float gain_offset, float eps,
                            void* out, double* lo, double* hi, double* mag) {
    if (!valid_dtype(in_dtype) || !valid_dtype(out_dtype) || rows < 0 || hidden <= 0 ||
        (rows && (!x || !out)))
        return -1;
    for (int64_t r = 0; r < rows; ++r) {
        const int64_t base = r * hidden;
        double ss = 0.0;
        for (int64_t j = 0; j < hidden; ++j) {
            double xj = load_elem(in_dtype, x, base + j);
            ss += xj * xj;
        }
        const double inv = inv_rms(ss, hidden, eps);
        for (int64_t j = 0; j < hidden; ++j) {
            double y = load_elem(in_dtype, x, base + j) * inv;
            if (gain) y *= eff_gain(gain, gain_offset, j);
            store_elem(out_dtype, out, base + j, y);
            put_check(lo, hi, mag, base + j, y, y, fabs(y));
        }
    }
    return 0;
}

/* Per-expert form of core 1 (MuseSparkMoE.pre_expert_norm /
 * post_expert_norm: per-expert norms over the tokens routed to each expert).
 * Rows [offsets[g], offsets[g+1]) are normalised with the gain row g of
 * gains [num_groups, hidden]; offsets has num_groups + 1 entries, starts at
 * 0, does not decrease and ends at rows. */
int muse_oracle_rms_norm_grouped(int dtype, const void* x, int64_t rows, int64_t hidden,
                                 const float* gains, float gain_offset, const int32_t* offsets,
                                 int32_t num_groups, float eps, void* out, double* lo, double* hi,
                                 double* mag) {
    if (!valid_dtype(dtype) || rows < 0 || hidden <= 0 || num_groups < 1 || !offsets || !gains)
        return -1;
    if (offsets[0] != 0 || offsets[num_groups] != rows) return -1;
    const size_t es = dtype == DT_BF16 ? 2 : 4;
    for (int32_t g = 0; g < num_groups; ++g) {
        const int64_t r0 = offsets[g], r1 = offsets[g + 1];
        if (r1 < r0) return -1;
        if (r1 == r0) continue;
        const int64_t e0 = r0 * hidden;
        const int rc = muse_oracle_rms_norm(
            dtype, (const char*)x + (size_t)e0 * es, r1 - r0, hidden, gains + (int64_t)g * hidden,
            gain_offset, eps, (char*)out + (size_t)e0 * es, lo ? lo + e0 : NULL, hi ? hi + e0 : NULL,
            mag ? mag + e0 : NULL);
        if (rc != 0) return rc;
    }
    return 0;
}

/* ------------------------------------------------------------------ core 2 */

/* _input_scale_norm_core: apply the effective gain first, then a
 * parameter-free RMS normalisation whose eps is added to the mean square of
 * the scaled activation. */
int muse_oracle_input_scale_norm(int dtype, const void* x, int64_t rows, int64_t hidden,
                                 const float* gain, float gain_offset, float eps,
                                 void* out, double* lo, double* hi, double* mag) {
    if (!valid_dtype(dtype) || rows < 0 || hidden <= 0 || (rows && (!x || !out))) return -1;
    for (int64_t r = 0; r < rows; ++r) {
        const int64_t base = r * hidden;
        double ss = 0.0;
        for (int64_t j = 0; j < hidden; ++j) {
            double z = load_elem(dtype, x, base + j) * eff_gain(gain, gain_offset, j);
            ss += z * z;
        }
        const double inv = inv_rms(ss, hidden, eps);
        for (int64_t j = 0; j < hidden; ++j) {
            double z = load_elem(dtype, x, base + j) * eff_gain(gain, gain_offset, j);
            double y = z * inv;
            store_elem(dtype, out, base + j, y);
            put_check(lo, hi, mag, base + j, y, y, fabs(y));
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ core 3 */

#define MAXC 4 /* a value with up to two casts in doubt has at most 4 candidates */

typedef struct {
    int n;
    double v[MAXC];
} cand_set;

static void cand_add(cand_set* s, double v) {
    for (int i = 0; i < s->n; ++i)
        if (s->v[i] == v) return;
    if (s->n < MAXC) s->v[s->n++] = v;
}

/* One head of core 3: normalise `width` elements of x over the head, cast,
 * and (query heads) scale and cast again.  Fills the candidate set of each
 * element; element j's primary value is cs[j].v[0]. */
static void qk_head_norm(int dtype, const void* x, int64_t base, int32_t d, float eps,
                         int is_query, float query_scale, cand_set* cs) {
    double ss = 0.0;
    for (int32_t j = 0; j < d; ++j) {
        double xj = load_elem(dtype, x, base + j);
        ss += xj * xj;
    }
    const double inv = inv_rms(ss, d, eps);
    for (int32_t j = 0; j < d; ++j) {
        double c[2];
        int nc = cast_candidates(dtype, load_elem(dtype, x, base + j) * inv, c);
        cand_set s = {0, {0}};
        if (!is_query) {
            for (int i = 0; i < nc; ++i) cand_add(&s, c[i]);
        } else {
            /* query_scale multiplies the query after its cast to the Q dtype;
             * the scaled value is cast to the Q dtype again. */
            for (int i = 0; i < nc; ++i) {
                double c2[2];
                int n2 = cast_candidates(dtype, c[i] * (double)query_scale, c2);
                for (int k = 0; k < n2; ++k) cand_add(&s, c2[k]);
            }
        }
        cs[j] = s;
    }
}

static void minmax_upd(double v, double* mn, double* mx) {
    if (v < *mn) *mn = v;
    if (v > *mx) *mx = v;
}

/* Rotate one head's normalised pairs and write outputs + check arrays. */
static void qk_head_out(int dtype, const cand_set* cs, int32_t d, const float* inv_freq,
                        int32_t pos, int use_rope, int upcast_rope, void* out,
                        double* lo, double* hi, double* mag, int64_t base) {
    if (!use_rope) {
        for (int32_t j = 0; j < d; ++j) {
            double mn = INFINITY, mx = -INFINITY;
            for (int i = 0; i < cs[j].n; ++i) minmax_upd(cs[j].v[i], &mn, &mx);
            store_elem(dtype, out, base + j, cs[j].v[0]);
            put_check(lo, hi, mag, base + j, mn, mx, fabs(cs[j].v[0]));
        }
        return;
    }
    const int fp32_rotation = upcast_rope || dtype == DT_F32;
    for (int32_t i = 0; i < d / 2; ++i) {
        const cand_set* A = &cs[2 * i];
        const cand_set* B = &cs[2 * i + 1];
        /* Angle in FP32: f32(pos) times the FP32 frequency, one FP32 rounding. */
        const float phi = (float)pos * inv_freq[i];
        const double c = cos((double)phi), s = sin((double)phi);
        double mn0 = INFINITY, mx0 = -INFINITY, mn1 = INFINITY, mx1 = -INFINITY;
        double m0 = 0.0, m1 = 0.0, y0p = 0.0, y1p = 0.0;
        if (fp32_rotation) {
            /* Legacy (original checkpoint) rotation: FP32 arithmetic. */
            for (int ia = 0; ia < A->n; ++ia)
                for (int ib = 0; ib < B->n; ++ib) {
                    const double a = A->v[ia], b = B->v[ib];
                    const double y0 = a * c - b * s;
                    const double y1 = a * s + b * c;
                    minmax_upd(y0, &mn0, &mx0);
                    minmax_upd(y1, &mn1, &mx1);
                    m0 = fmax(m0, fabs(a * c) + fabs(b * s));
                    m1 = fmax(m1, fabs(a * s) + fabs(b * c));
                    if (ia == 0 && ib == 0) { y0p = y0; y1p = y1; }
                }
        } else {
            /* v2 (HF release) rotation in the Q/K dtype: cos/sin are cast to
             * it, each of the two products is rounded to it before the
             * addition, and the sum is cast once more.  Every step after the
             * candidate casts is exact in FP32, so mag stays 0. */
            double C[2], S[2];
            const int nC = cast_candidates(dtype, c, C);
            const int nS = cast_candidates(dtype, s, S);
            for (int ia = 0; ia < A->n; ++ia)
                for (int ib = 0; ib < B->n; ++ib)
                    for (int ic = 0; ic < nC; ++ic)
                        for (int is = 0; is < nS; ++is) {
                            const double a = A->v[ia], b = B->v[ib];
                            const double y0 = cast_to(dtype, a * C[ic]) - cast_to(dtype, b * S[is]);
                            const double y1 = cast_to(dtype, a * S[is]) + cast_to(dtype, b * C[ic]);
                            minmax_upd(y0, &mn0, &mx0);
                            minmax_upd(y1, &mn1, &mx1);
                            if (ia == 0 && ib == 0 && ic == 0 && is == 0) { y0p = y0; y1p = y1; }
                        }
        }
        store_elem(dtype, out, base + 2 * i, y0p);
        store_elem(dtype, out, base + 2 * i + 1, y1p);
        put_check(lo, hi, mag, base + 2 * i, mn0, mx0, m0);
        put_check(lo, hi, mag, base + 2 * i + 1, mn1, mx1, m1);
    }
}

/* _qk_norm_rope_core: per-head FP32 RMS normalisation of Q and K cast back to
 * their dtype, query_scale after the query's cast, then adjacent-pair RoPE
 * (pairs (2i, 2i+1), the native checkpoint's convention) in FP32 (legacy) or
 * in the Q/K dtype (v2).  K is never scaled. */
int muse_oracle_qk_norm_rope(int dtype, const void* q, const void* k, int64_t tokens,
                             int32_t hq, int32_t hkv, int32_t head_dim,
                             const int32_t* pos, float eps, float query_scale,
                             int use_rope, int upcast_rope, float rope_base,
                             void* q_out, double* q_lo, double* q_hi, double* q_mag,
                             void* k_out, double* k_lo, double* k_hi, double* k_mag) {
    if (!valid_dtype(dtype) || tokens < 0 || hq <= 0 || hkv <= 0 || head_dim <= 0 ||
        (head_dim & 1))
        return -1;
    if (tokens && (!q || !k || !q_out || !k_out || (use_rope && !pos))) return -1;
    float* inv_freq = (float*)malloc(sizeof(float) * (size_t)(head_dim / 2));
    cand_set* cs = (cand_set*)malloc(sizeof(cand_set) * (size_t)head_dim);
    if (!inv_freq || !cs) { free(inv_freq); free(cs); return -1; }
    if (use_rope && muse_oracle_inv_freq(head_dim, rope_base, inv_freq) != 0) {
        free(inv_freq); free(cs); return -1;
    }
    for (int64_t t = 0; t < tokens; ++t) {
        const int32_t p = use_rope ? pos[t] : 0;
        for (int32_t h = 0; h < hq; ++h) {
            const int64_t base = (t * hq + h) * (int64_t)head_dim;
            qk_head_norm(dtype, q, base, head_dim, eps, 1, query_scale, cs);
            qk_head_out(dtype, cs, head_dim, inv_freq, p, use_rope, upcast_rope, q_out,
                        q_lo, q_hi, q_mag, base);
        }
        for (int32_t h = 0; h < hkv; ++h) {
            const int64_t base = (t * hkv + h) * (int64_t)head_dim;
            qk_head_norm(dtype, k, base, head_dim, eps, 0, 1.0f, cs);
            qk_head_out(dtype, cs, head_dim, inv_freq, p, use_rope, upcast_rope, k_out,
                        k_lo, k_hi, k_mag, base);
        }
    }
    free(inv_freq);
    free(cs);
    return 0;
}

/* ------------------------------------------------------------------ core 4 */

/* _output_norm_gate_core: parameter-free RMS normalisation of the attention
 * output times the sigmoid of the gate projection, both in FP32, one cast to
 * the original dtype. */
int muse_oracle_output_norm_gate(int dtype, const void* o, const void* g, int64_t tokens,
                                 int32_t heads, int32_t head_dim, int32_t norm_group,
                                 float eps, void* out, double* lo, double* hi, double* mag) {
    if (!valid_dtype(dtype) || tokens < 0 || heads <= 0 || head_dim <= 0) return -1;
    const int64_t width = (int64_t)heads * head_dim;
    if (norm_group != head_dim && norm_group != width) return -1;
    if (tokens && (!o || !g || !out)) return -1;
    const int64_t groups = tokens * width / norm_group;
    for (int64_t gi = 0; gi < groups; ++gi) {
        const int64_t base = gi * norm_group;
        double ss = 0.0;
        for (int32_t j = 0; j < norm_group; ++j) {
            double oj = load_elem(dtype, o, base + j);
            ss += oj * oj;
        }
        const double inv = inv_rms(ss, norm_group, eps);
        for (int32_t j = 0; j < norm_group; ++j) {
            const double sig = 1.0 / (1.0 + exp(-load_elem(dtype, g, base + j)));
            const double y = load_elem(dtype, o, base + j) * inv * sig;
            store_elem(dtype, out, base + j, y);
            put_check(lo, hi, mag, base + j, y, y, fabs(y));
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ core 5 */

/* _norm_residual_core with the declared learned blend
 * h' = cos(theta) * h + sin(theta) * nb: the branch is normalised (gain after
 * the norm, or before it when input_scale is set), cast back to the branch
 * dtype before the blend (the branch cast is left unchanged by the fusion),
 * then blended into the FP32 stream per channel. */
int muse_oracle_norm_residual(const float* stream, int branch_dtype, const void* branch,
                              int64_t rows, int64_t hidden, const float* gain,
                              float gain_offset, const float* theta, int input_scale,
                              float norm_eps, float* out, double* lo, double* hi,
                              double* mag) {
    if (!valid_dtype(branch_dtype) || rows < 0 || hidden <= 0) return -1;
    if (rows && (!stream || !branch || !out || !theta)) return -1;
    for (int64_t r = 0; r < rows; ++r) {
        const int64_t base = r * hidden;
        double ss = 0.0;
        for (int64_t j = 0; j < hidden; ++j) {
            double b = load_elem(branch_dtype, branch, base + j);
            if (input_scale) b *= eff_gain(gain, gain_offset, j);
            ss += b * b;
        }
        const double inv = inv_rms(ss, hidden, norm_eps);
        for (int64_t j = 0; j < hidden; ++j) {
            const double b = load_elem(branch_dtype, branch, base + j);
            const double w = eff_gain(gain, gain_offset, j);
            const double v = input_scale ? (b * w) * inv : (b * inv) * w;
            double nb[2];
            const int n = cast_candidates(branch_dtype, v, nb);
            const double c = cos((double)theta[j]), s = sin((double)theta[j]);
            const double h = (double)stream[base + j];
            double mn = INFINITY, mx = -INFINITY, m = 0.0;
            for (int i = 0; i < n; ++i) {
                const double y = c * h + s * nb[i];
                minmax_upd(y, &mn, &mx);
                m = fmax(m, fabs(c * h) + fabs(s * nb[i]));
            }
            out[base + j] = (float)(c * h + s * nb[0]);
            put_check(lo, hi, mag, base + j, mn, mx, m);
        }
    }
    return 0;
}

/* -------------------------------------------------- _residual_core (blend) */

/* _residual_core / MuseSparkResidual.forward: the residual stream blended
 * with the branch as it arrives (no branch norm), under the declared blend of
 * core 5: out = cos(theta) h + sin(theta) branch per channel, FP32 theta, the
 * branch read exactly in double (bf16 -> f32 is exact), the stream dtype kept. */
int muse_oracle_residual_blend(const float* stream, int branch_dtype, const void* branch,
                               int64_t rows, int64_t hidden, const float* theta, float* out,
                               double* lo, double* hi, double* mag) {
    if (!valid_dtype(branch_dtype) || rows < 0 || hidden <= 0) return -1;
    if (rows && (!stream || !branch || !out || !theta)) return -1;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t j = 0; j < hidden; ++j) {
            const int64_t i = r * hidden + j;
            const double c = cos((double)theta[j]), s = sin((double)theta[j]);
            const double h = (double)stream[i], b = load_elem(branch_dtype, branch, i);
            const double y = c * h + s * b;
            out[i] = (float)y;
            put_check(lo, hi, mag, i, y, y, fabs(c * h) + fabs(s * b));
        }
    }
    return 0;
}

/* The learned gate of _residual_core / MuseSparkResidual (gate [hidden],
 * temperature, eps) as the blend's two coefficients - the declared reading:
 * the squared residual coefficient is the sigmoid of gate / temperature,
 * bounded below by eps ("lower bound on the squared residual coefficient"),
 * and the branch coefficient keeps the squares summing to one
 * ("norm-preserving"):
 *   c^2 = max(sigmoid(gate / temperature), eps),   s^2 = 1 - c^2,
 * c, s >= 0, so that theta = atan2(s, c) lies in [0, pi/2] and the blend is
 * core 5's cos(theta) h + sin(theta) b.  1 - max(sigmoid(x), eps) is written
 * as min(sigmoid(-x), 1 - eps), the same number, so that s keeps its
 * relative precision when sigmoid(x) is close to 1.  Any of c, s, theta may
 * be NULL. */
int muse_oracle_residual_gate_coefficients(const float* gate, int64_t hidden, float temperature,
                                           float eps, double* c, double* s, double* theta) {
    if (!gate || hidden <= 0 || !(temperature > 0.0f) || !(eps >= 0.0f && eps <= 1.0f)) return -1;
    for (int64_t j = 0; j < hidden; ++j) {
        const double x = (double)gate[j] / (double)temperature;
        const double c2 = fmax(1.0 / (1.0 + exp(-x)), (double)eps);
        const double s2 = fmin(1.0 / (1.0 + exp(x)), 1.0 - (double)eps);
        const double cj = sqrt(c2), sj = sqrt(s2);
        if (c) c[j] = cj;
        if (s) s[j] = sj;
        if (theta) theta[j] = atan2(sj, cj);
    }
    return 0;
}

/* _residual_core(stream, branch, gate, temperature, eps) under the reading
 * above: out = c h + s branch per channel. */
int muse_oracle_residual(const float* stream, int branch_dtype, const void* branch, int64_t rows,
                         int64_t hidden, const float* gate, float temperature, float eps, float* out,
                         double* lo, double* hi, double* mag) {
    if (!valid_dtype(branch_dtype) || rows < 0 || hidden <= 0 || !gate) return -1;
    if (rows && (!stream || !branch || !out)) return -1;
    double* c = (double*)malloc(sizeof(double) * (size_t)hidden);
    double* s = (double*)malloc(sizeof(double) * (size_t)hidden);
    if (!c || !s || muse_oracle_residual_gate_coefficients(gate, hidden, temperature, eps, c, s, NULL)) {
        free(c);
        free(s);
        return -1;
    }
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t j = 0; j < hidden; ++j) {
            const int64_t i = r * hidden + j;
            const double h = (double)stream[i], b = load_elem(branch_dtype, branch, i);
            const double y = c[j] * h + s[j] * b;
            out[i] = (float)y;
            put_check(lo, hi, mag, i, y, y, fabs(c[j] * h) + fabs(s[j] * b));
        }
    }
    free(c);
    free(s);
    return 0;
}

/* ================================================================ backward
 *
 * The cores run under autograd (the page's _checkpoint_recomputed_math keeps
 * them outside checkpoint caching while "autograd ... still run[s]").  Their
 * backward is therefore the derivative of the forward map above, evaluated
 * from the saved forward inputs with r recomputed, where every dtype boundary
 * the forward materialises passes the gradient through and rounds it to that
 * tensor's dtype (the gradient of a cast is the incoming gradient cast back):
 *   - the output cast of each core: dy arrives in the output dtype;
 *   - core 3: the gradient of the normalised Q/K (and of the scaled query) is
 *     rounded to the Q/K dtype;
 *   - core 5: the gradient of the cast branch nb is rounded to the branch
 *     dtype;
 *   - input gradients are cast once to the input dtype; parameter gradients
 *     (gain, theta) are FP32 sums over all rows.
 * round_grads = 0 drops the intermediate roundings (the exact derivative;
 * used by the pins).
 *
 * Check arrays: as for the forward, lo/hi bracket the exact pre-cast value
 * over the admissible values of every intermediate cast (forward casts whose
 * values enter the gradient, and gradient casts), and mag is the sum of the
 * magnitudes of the terms of the last expression, with each inner sum
 * counted by the magnitudes of its own terms.  Parameter gradients come as
 * [lo, hi] and mag over the row sum.
 */

typedef struct {
    double lo, hi, rn; /* bracket and the round-to-nearest path value */
    double m;          /* magnitude its FP32 evaluation error is relative to */
} ival;

static ival iv_exact(double v) { ival r = {v, v, v, fabs(v)}; return r; }

static ival iv_cast(int dtype, double v, int round) {
    if (!round) return iv_exact(v);
    double c[2];
    const int n = cast_candidates(dtype, v, c);
    ival r = {c[0], c[0], c[0], fabs(c[0])};
    if (n == 2) { r.lo = fmin(c[0], c[1]); r.hi = fmax(c[0], c[1]); r.m = fmax(fabs(r.lo), fabs(r.hi)); }
    return r;
}

/* A cast whose argument is an FP32-evaluated sum of terms of total magnitude
 * `terms`: its evaluation error is relative to `terms`, not to the possibly
 * cancelling value, so every bf16 value within 2^-20 * max(|v|, terms) of v
 * is an admissible result (the rule of cast_candidates with the sum's own
 * magnitude); an FP32 cast keeps one value and carries `terms` forward as
 * the magnitude later allowances scale with. */
static ival iv_cast_sum(int dtype, double v, double terms, int round) {
    const double m = fmax(fabs(v), terms);
    if (!round) { ival r = {v, v, v, m}; return r; }
    if (dtype != DT_BF16) { const double f = cast_to(dtype, v); ival r = {f, f, f, m}; return r; }
    const double d = m * MUSE_ORACLE_AMBIG_REL;
    ival r = {bf16_round(v - d), bf16_round(v + d), bf16_round(v), 0.0};
    r.m = fmax(fabs(r.lo), fabs(r.hi));
    return r;
}

/* interval times a real scalar */
static ival iv_scale(ival a, double s) {
    ival r;
    r.rn = a.rn * s;
    const double p = a.lo * s, q = a.hi * s;
    r.lo = fmin(p, q);
    r.hi = fmax(p, q);
    r.m = a.m * fabs(s);
    return r;
}

static ival iv_add(ival a, ival b) {
    ival r = {a.lo + b.lo, a.hi + b.hi, a.rn + b.rn, a.m + b.m};
    return r;
}

static double iv_absmax(ival a) { return fmax(fabs(a.lo), fabs(a.hi)); }

/* Gradient of one normalised row.  mode 0 (core 1 form): y = x r(x) w;
 * mode 1 (core 2 form): z = x w, y = z r(z).  g = dL/dy per element (an
 * interval when it passed a rounded cast).  Fills dx (interval + mag) and, if
 * dw_term is not NULL, each row's term of the gain gradient.
 *   mode 0: dx_k = r w_k g_k - r^3 x_k C / H,  C = sum_j g_j w_j x_j;
 *           dW_k += g_k x_k r
 *   mode 1: dz_k = r g_k - r^3 z_k C / H,      C = sum_j g_j z_j;
 *           dx_k = dz_k w_k;                    dW_k += dz_k x_k */
static void norm_row_bwd(int mode, int64_t H, const double* x, const double* w, float eps,
                         const ival* g, ival* dx, double* dx_mag, ival* dw_term,
                         double* dw_mag) {
    double ss = 0.0;
    for (int64_t j = 0; j < H; ++j) {
        const double u = mode ? x[j] * w[j] : x[j];
        ss += u * u;
    }
    const double r = inv_rms(ss, H, eps);
    const double r3 = r * r * r;
    ival C = iv_exact(0.0);
    double Cabs = 0.0;
    for (int64_t j = 0; j < H; ++j) {
        const double f = mode ? x[j] * w[j] : w[j] * x[j];
        C = iv_add(C, iv_scale(g[j], f));
        Cabs += g[j].m * fabs(f);
    }
    for (int64_t k = 0; k < H; ++k) {
        const double u = mode ? x[k] * w[k] : x[k];
        const double a = mode ? r : r * w[k];
        ival d = iv_add(iv_scale(g[k], a), iv_scale(C, -r3 * u / (double)H));
        double m = g[k].m * fabs(a) + r3 * fabs(u) * Cabs / (double)H;
        if (mode) {
            if (dw_term) {
                dw_term[k] = iv_scale(d, x[k]);
                dw_mag[k] = m * fabs(x[k]);
            }
            d = iv_scale(d, w[k]);
            m *= fabs(w[k]);
        } else if (dw_term) {
            dw_term[k] = iv_scale(g[k], x[k] * r);
            dw_mag[k] = g[k].m * fabs(x[k] * r);
        }
        dx[k] = d;
        dx_mag[k] = m;
    }
}

static void acc_param(double* lo, double* hi, double* mag, int64_t k, ival t, double m) {
    if (lo) lo[k] += t.lo;
    if (hi) hi[k] += t.hi;
    if (mag) mag[k] += m;
}

static void zero_n(double* p, int64_t n) {
    if (p) memset(p, 0, sizeof(double) * (size_t)n);
}

static int rows_bwd(int mode, int dtype, const void* x, const void* dy, int64_t rows,
                    int64_t hidden, const float* gain, float gain_offset, float eps, void* dx,
                    double* lo, double* hi, double* mag, double* dgain_lo, double* dgain_hi,
                    double* dgain_mag) {
    if (!valid_dtype(dtype) || rows < 0 || hidden <= 0 || (rows && (!x || !dy || !dx))) return -1;
    double* xv = (double*)malloc(sizeof(double) * (size_t)hidden * 3);
    ival* g = (ival*)malloc(sizeof(ival) * (size_t)hidden * 3);
    double* dm = (double*)malloc(sizeof(double) * (size_t)hidden * 2);
    if (!xv || !g || !dm) { free(xv); free(g); free(dm); return -1; }
    double* w = xv + hidden;
    ival* d = g + hidden;
    ival* wt = g + 2 * hidden;
    double* wm = dm + hidden;
    for (int64_t j = 0; j < hidden; ++j) w[j] = eff_gain(gain, gain_offset, j);
    zero_n(dgain_lo, hidden);
    zero_n(dgain_hi, hidden);
    zero_n(dgain_mag, hidden);
    for (int64_t r = 0; r < rows; ++r) {
        const int64_t base = r * hidden;
        for (int64_t j = 0; j < hidden; ++j) {
            xv[j] = load_elem(dtype, x, base + j);
            g[j] = iv_exact(load_elem(dtype, dy, base + j));
        }
        norm_row_bwd(mode, hidden, xv, w, eps, g, d, dm, gain ? wt : NULL, wm);
        for (int64_t j = 0; j < hidden; ++j) {
            store_elem(dtype, dx, base + j, d[j].rn);
            put_check(lo, hi, mag, base + j, d[j].lo, d[j].hi, dm[j]);
            if (gain) acc_param(dgain_lo, dgain_hi, dgain_mag, j, wt[j], wm[j]);
        }
    }
    free(xv);
    free(g);
    free(dm);
    return 0;
}

int muse_oracle_rms_norm_bwd(int dtype, const void* x, const void* dy, int64_t rows,
                             int64_t hidden, const float* gain, float gain_offset, float eps,
                             void* dx, double* lo, double* hi, double* mag, double* dgain_lo,
                             double* dgain_hi, double* dgain_mag) {
    return rows_bwd(0, dtype, x, dy, rows, hidden, gain, gain_offset, eps, dx, lo, hi, mag,
                    dgain_lo, dgain_hi, dgain_mag);
}

int muse_oracle_input_scale_norm_bwd(int dtype, const void* x, const void* dy, int64_t rows,
                                     int64_t hidden, const float* gain, float gain_offset,
                                     float eps, void* dx, double* lo, double* hi, double* mag,
                                     double* dgain_lo, double* dgain_hi, double* dgain_mag) {
    return rows_bwd(1, dtype, x, dy, rows, hidden, gain, gain_offset, eps, dx, lo, hi, mag,
                    dgain_lo, dgain_hi, dgain_mag);
}

/* sigmoid'(v) = e^-|v| / (1 + e^-|v|)^2 (the form without cancellation). */
static double dsigmoid(double v) {
    const double t = exp(-fabs(v));
    return t / ((1.0 + t) * (1.0 + t));
}

int muse_oracle_output_norm_gate_bwd(int dtype, const void* o, const void* g, const void* dy,
                                     int64_t tokens, int32_t heads, int32_t head_dim,
                                     int32_t norm_group, float eps, void* d_o, double* do_lo,
                                     double* do_hi, double* do_mag, void* dg, double* dg_lo,
                                     double* dg_hi, double* dg_mag) {
    if (!valid_dtype(dtype) || tokens < 0 || heads <= 0 || head_dim <= 0) return -1;
    const int64_t width = (int64_t)heads * head_dim;
    if (norm_group != head_dim && norm_group != width) return -1;
    if (tokens && (!o || !g || !dy || !d_o || !dg)) return -1;
    double* ov = (double*)malloc(sizeof(double) * (size_t)norm_group * 3);
    ival* gr = (ival*)malloc(sizeof(ival) * (size_t)norm_group * 2);
    if (!ov || !gr) { free(ov); free(gr); return -1; }
    double* one = ov + norm_group;
    double* dm = ov + 2 * (int64_t)norm_group;
    ival* dd = gr + norm_group;
    for (int32_t j = 0; j < norm_group; ++j) one[j] = 1.0;
    const int64_t groups = tokens * width / norm_group;
    for (int64_t gi = 0; gi < groups; ++gi) {
        const int64_t base = gi * norm_group;
        double ss = 0.0;
        for (int32_t j = 0; j < norm_group; ++j) {
            ov[j] = load_elem(dtype, o, base + j);
            ss += ov[j] * ov[j];
        }
        const double r = inv_rms(ss, norm_group, eps);
        for (int32_t j = 0; j < norm_group; ++j) {
            const double gv = load_elem(dtype, g, base + j);
            const double dyv = load_elem(dtype, dy, base + j);
            const double s = 1.0 / (1.0 + exp(-gv));
            gr[j] = iv_exact(dyv * s); /* dL/dn, n = o r */
            const double dgv = dyv * ov[j] * r * dsigmoid(gv);
            store_elem(dtype, dg, base + j, dgv);
            put_check(dg_lo, dg_hi, dg_mag, base + j, dgv, dgv, fabs(dgv));
        }
        norm_row_bwd(0, norm_group, ov, one, eps, gr, dd, dm, NULL, NULL);
        for (int32_t j = 0; j < norm_group; ++j) {
            store_elem(dtype, d_o, base + j, dd[j].rn);
            put_check(do_lo, do_hi, do_mag, base + j, dd[j].lo, dd[j].hi, dm[j]);
        }
    }
    free(ov);
    free(gr);
    return 0;
}

int muse_oracle_norm_residual_bwd(const float* stream, int branch_dtype, const void* branch,
                                  const float* dstream_out, int64_t rows, int64_t hidden,
                                  const float* gain, float gain_offset, const float* theta,
                                  int input_scale, float norm_eps, int round_grads,
                                  float* dstream, double* ds_lo, double* ds_hi, double* ds_mag,
                                  void* dbranch, double* db_lo, double* db_hi, double* db_mag,
                                  double* dgain_lo, double* dgain_hi, double* dgain_mag,
                                  double* dtheta_lo, double* dtheta_hi, double* dtheta_mag) {
    if (!valid_dtype(branch_dtype) || rows < 0 || hidden <= 0) return -1;
    if (rows && (!stream || !branch || !dstream_out || !theta || !dstream || !dbranch)) return -1;
    double* bv = (double*)malloc(sizeof(double) * (size_t)hidden * 4);
    ival* gr = (ival*)malloc(sizeof(ival) * (size_t)hidden * 3);
    if (!bv || !gr) { free(bv); free(gr); return -1; }
    double* w = bv + hidden;
    double* dm = bv + 2 * hidden;
    double* wm = bv + 3 * hidden;
    ival* dd = gr + hidden;
    ival* wt = gr + 2 * hidden;
    const int mode = input_scale ? 1 : 0;
    for (int64_t j = 0; j < hidden; ++j) w[j] = eff_gain(gain, gain_offset, j);
    zero_n(dgain_lo, hidden);
    zero_n(dgain_hi, hidden);
    zero_n(dgain_mag, hidden);
    zero_n(dtheta_lo, hidden);
    zero_n(dtheta_hi, hidden);
    zero_n(dtheta_mag, hidden);
    for (int64_t r = 0; r < rows; ++r) {
        const int64_t base = r * hidden;
        double ss = 0.0;
        for (int64_t j = 0; j < hidden; ++j) {
            bv[j] = load_elem(branch_dtype, branch, base + j);
            const double u = mode ? bv[j] * w[j] : bv[j];
            ss += u * u;
        }
        const double inv = inv_rms(ss, hidden, norm_eps);
        for (int64_t j = 0; j < hidden; ++j) {
            const double c = cos((double)theta[j]), s = sin((double)theta[j]);
            const double dh = (double)dstream_out[base + j];
            const double h = (double)stream[base + j];
            /* dL/dh = cos(theta) dh' (FP32 output) */
            dstream[base + j] = (float)(c * dh);
            put_check(ds_lo, ds_hi, ds_mag, base + j, c * dh, c * dh, fabs(c * dh));
            /* dL/dnb = sin(theta) dh', rounded to the branch dtype */
            gr[j] = iv_cast(branch_dtype, s * dh, round_grads);
            /* dL/dtheta = dh' (-sin(theta) h + cos(theta) nb), nb the forward's cast value */
            const double v = mode ? (bv[j] * w[j]) * inv : (bv[j] * inv) * w[j];
            const ival nb = iv_cast(branch_dtype, v, 1);
            const ival t = iv_add(iv_exact(-s * h * dh), iv_scale(nb, c * dh));
            acc_param(dtheta_lo, dtheta_hi, dtheta_mag, j, t,
                      fabs(dh) * (fabs(s * h) + fabs(c) * iv_absmax(nb)));
        }
        norm_row_bwd(mode, hidden, bv, w, norm_eps, gr, dd, dm, gain ? wt : NULL, wm);
        for (int64_t j = 0; j < hidden; ++j) {
            store_elem(branch_dtype, dbranch, base + j, dd[j].rn);
            put_check(db_lo, db_hi, db_mag, base + j, dd[j].lo, dd[j].hi, dm[j]);
            if (gain) acc_param(dgain_lo, dgain_hi, dgain_mag, j, wt[j], wm[j]);
        }
    }
    free(bv);
    free(gr);
    return 0;
}

/* Backward of _residual_core, both forms: out = c h + s b per channel (b the
 * branch read in FP32).  Given dy = dL/dout (FP32):
 *   dstream = c dy                          (FP32);
 *   dbranch = cast_branch(s dy)             (the forward upcast the branch to
 *                                            FP32; the gradient of that cast
 *                                            is rounded back);
 *   angle form: dtheta_j = sum over rows of dy (-s h + c b),
 *               c = cos(theta_j), s = sin(theta_j);
 *   gate form:  dgate_j  = sum over rows of dy (c' h + s' b), with
 *               c' = dc/dgate = c s^2 / (2 temperature),
 *               s' = ds/dgate = -s c^2 / (2 temperature)
 *               where sigmoid(gate / temperature) >= eps (c^2 = sigmoid there),
 *               and c' = s' = 0 where the bound holds c (clamp_min's rule: the
 *               gradient passes at equality).
 * Parameter gradients come as (lo, hi, mag): the exact sum twice and the sum
 * of the magnitudes of its terms. */
static int residual_bwd(const float* stream, int branch_dtype, const void* branch, const float* dy,
                        int64_t rows, int64_t hidden, const double* c, const double* s,
                        const double* dc, const double* ds, float* dstream, double* ds_lo,
                        double* ds_hi, double* ds_mag, void* dbranch, double* db_lo, double* db_hi,
                        double* db_mag, double* dp_lo, double* dp_hi, double* dp_mag) {
    if (rows && (!stream || !branch || !dy || !dstream || !dbranch)) return -1;
    zero_n(dp_lo, hidden);
    zero_n(dp_hi, hidden);
    zero_n(dp_mag, hidden);
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t j = 0; j < hidden; ++j) {
            const int64_t i = r * hidden + j;
            const double g = (double)dy[i], h = (double)stream[i];
            const double b = load_elem(branch_dtype, branch, i);
            dstream[i] = (float)(c[j] * g);
            put_check(ds_lo, ds_hi, ds_mag, i, c[j] * g, c[j] * g, fabs(c[j] * g));
            store_elem(branch_dtype, dbranch, i, s[j] * g);
            put_check(db_lo, db_hi, db_mag, i, s[j] * g, s[j] * g, fabs(s[j] * g));
            const double t = g * (dc[j] * h + ds[j] * b);
            acc_param(dp_lo, dp_hi, dp_mag, j, iv_exact(t), fabs(g) * (fabs(dc[j] * h) + fabs(ds[j] * b)));
        }
    }
    return 0;
}

int muse_oracle_residual_blend_bwd(const float* stream, int branch_dtype, const void* branch,
                                   const float* dy, int64_t rows, int64_t hidden, const float* theta,
                                   float* dstream, double* ds_lo, double* ds_hi, double* ds_mag,
                                   void* dbranch, double* db_lo, double* db_hi, double* db_mag,
                                   double* dtheta_lo, double* dtheta_hi, double* dtheta_mag) {
    if (!valid_dtype(branch_dtype) || rows < 0 || hidden <= 0 || !theta) return -1;
    double* cs = (double*)malloc(sizeof(double) * (size_t)hidden * 4);
    if (!cs) return -1;
    double *c = cs, *s = cs + hidden, *dc = cs + 2 * hidden, *ds = cs + 3 * hidden;
    for (int64_t j = 0; j < hidden; ++j) {
        c[j] = cos((double)theta[j]);
        s[j] = sin((double)theta[j]);
        dc[j] = -s[j]; /* d cos / d theta */
        ds[j] = c[j];  /* d sin / d theta */
    }
    const int rc = residual_bwd(stream, branch_dtype, branch, dy, rows, hidden, c, s, dc, ds, dstream,
                                ds_lo, ds_hi, ds_mag, dbranch, db_lo, db_hi, db_mag, dtheta_lo,
                                dtheta_hi, dtheta_mag);
    free(cs);
    return rc;
}

int muse_oracle_residual_bwd(const float* stream, int branch_dtype, const void* branch,
                             const float* dy, int64_t rows, int64_t hidden, const float* gate,
                             float temperature, float eps, float* dstream, double* ds_lo,
                             double* ds_hi, double* ds_mag, void* dbranch, double* db_lo,
                             double* db_hi, double* db_mag, double* dgate_lo, double* dgate_hi,
                             double* dgate_mag) {
    if (!valid_dtype(branch_dtype) || rows < 0 || hidden <= 0 || !gate) return -1;
    double* cs = (double*)malloc(sizeof(double) * (size_t)hidden * 4);
    if (!cs) return -1;
    double *c = cs, *s = cs + hidden, *dc = cs + 2 * hidden, *ds = cs + 3 * hidden;
    if (muse_oracle_residual_gate_coefficients(gate, hidden, temperature, eps, c, s, NULL)) {
        free(cs);
        return -1;
    }
    for (int64_t j = 0; j < hidden; ++j) {
        const double x = (double)gate[j] / (double)temperature;
        const int free_ = 1.0 / (1.0 + exp(-x)) >= (double)eps;
        dc[j] = free_ ? c[j] * s[j] * s[j] / (2.0 * (double)temperature) : 0.0;
        ds[j] = free_ ? -s[j] * c[j] * c[j] / (2.0 * (double)temperature) : 0.0;
    }
    const int rc = residual_bwd(stream, branch_dtype, branch, dy, rows, hidden, c, s, dc, ds, dstream,
                                ds_lo, ds_hi, ds_mag, dbranch, db_lo, db_hi, db_mag, dgate_lo,
                                dgate_hi, dgate_mag);
    free(cs);
    return rc;
}

/* Gradient of one pair's rotated-in values under the v2 rotation (bf16):
 * the forward's y0 = cast(cast(a C) - cast(b S)), y1 = cast(cast(a S) +
 * cast(b C)) with C = cast(c), S = cast(s).  Backward through those bf16
 * operations: each product's gradient is the incoming gradient times the
 * other factor, rounded to bf16, and the two gradients reaching a (or b) are
 * added in bf16:
 *   da = cast(cast(dy0 C) + cast(dy1 S)),   db = cast(cast(dy1 C) - cast(dy0 S));
 * then, for query heads, cast(. * query_scale).  Products of two bf16 values
 * are exact; the sums and the scaling take cast_candidates' values; C and S
 * each take theirs (an FP32 sine or cosine near a bf16 midpoint). */
static void qk_pair_bwd_v2(int dtype, double y0, double y1, float phi, int is_query,
                           float query_scale, ival out[2]) {
    double C[2], S[2];
    const int nC = cast_candidates(dtype, cos((double)phi), C);
    const int nS = cast_candidates(dtype, sin((double)phi), S);
    for (int e = 0; e < 2; ++e) {
        double mn = INFINITY, mx = -INFINITY, prim = 0.0;
        for (int ic = 0; ic < nC; ++ic)
            for (int is = 0; is < nS; ++is) {
                const double v = e == 0 ? cast_to(dtype, y0 * C[ic]) + cast_to(dtype, y1 * S[is])
                                        : cast_to(dtype, y1 * C[ic]) - cast_to(dtype, y0 * S[is]);
                double g[2];
                const int ng = cast_candidates(dtype, v, g);
                for (int ig = 0; ig < ng; ++ig) {
                    double h[2] = {g[ig], g[ig]};
                    int nh = 1;
                    if (is_query) nh = cast_candidates(dtype, g[ig] * (double)query_scale, h);
                    for (int ih = 0; ih < nh; ++ih) minmax_upd(h[ih], &mn, &mx);
                    if (ic == 0 && is == 0 && ig == 0) prim = h[0];
                }
            }
        out[e].lo = mn;
        out[e].hi = mx;
        out[e].rn = prim;
        out[e].m = fmax(fabs(mn), fabs(mx));
    }
}

/* Core 3 backward.  Per head, FP32 (legacy) rotation:
 *   dm = R(phi)^T dy                     (FP32: da = c dy0 + s dy1, db = -s dy0 + c dy1)
 *   dn2 = cast(dm)                       (gradient of the rotated-in value, Q/K dtype)
 *   query heads: dn1 = cast(dn2 * query_scale); key heads: dn1 = dn2
 * or, v2 rotation on bf16 tensors, dn1 from qk_pair_bwd_v2; then
 *   dx = r dn1 - r^3 x (sum_j dn1_j x_j) / d, cast to the Q/K dtype. */
static void qk_head_bwd(int dtype, const void* x, const void* dy, int64_t base, int32_t d,
                        const float* inv_freq, int32_t pos, int use_rope, int v2, float eps,
                        int is_query, float query_scale, int round_grads, double* xv,
                        double* one, ival* gr, ival* dd, double* dm, void* dx, double* lo,
                        double* hi, double* mag) {
    for (int32_t j = 0; j < d; ++j) xv[j] = load_elem(dtype, x, base + j);
    for (int32_t i = 0; i < d / 2; ++i) {
        if (v2) {
            qk_pair_bwd_v2(dtype, load_elem(dtype, dy, base + 2 * i), load_elem(dtype, dy, base + 2 * i + 1),
                           (float)pos * inv_freq[i], is_query, query_scale, gr + 2 * i);
            continue;
        }
        double m0, m1;
        const double y0 = load_elem(dtype, dy, base + 2 * i);
        const double y1 = load_elem(dtype, dy, base + 2 * i + 1);
        if (use_rope) {
            const float phi = (float)pos * inv_freq[i];
            const double c = cos((double)phi), s = sin((double)phi);
            m0 = c * y0 + s * y1;
            m1 = -s * y0 + c * y1;
        } else {
            m0 = y0;
            m1 = y1;
        }
        const double m[2] = {m0, m1};
        /* magnitudes of the two products forming each component */
        double t[2] = {fabs(y0), fabs(y1)};
        if (use_rope) {
            const float phi = (float)pos * inv_freq[i];
            const double c = cos((double)phi), s = sin((double)phi);
            t[0] = fabs(c * y0) + fabs(s * y1);
            t[1] = fabs(s * y0) + fabs(c * y1);
        }
        for (int e = 0; e < 2; ++e) {
            const ival n2 = iv_cast_sum(dtype, m[e], t[e], round_grads);
            ival n1 = n2;
            if (is_query) {
                /* each admissible dn2 scaled, then cast again */
                const ival a = iv_cast(dtype, n2.lo * (double)query_scale, round_grads);
                const ival b = iv_cast(dtype, n2.hi * (double)query_scale, round_grads);
                const ival p = iv_cast(dtype, n2.rn * (double)query_scale, round_grads);
                n1.lo = fmin(fmin(a.lo, b.lo), fmin(a.hi, b.hi));
                n1.hi = fmax(fmax(a.lo, b.lo), fmax(a.hi, b.hi));
                n1.rn = p.rn;
                n1.m = fmax(n2.m * fabs((double)query_scale), fmax(fabs(n1.lo), fabs(n1.hi)));
            }
            gr[2 * i + e] = n1;
        }
    }
    norm_row_bwd(0, d, xv, one, eps, gr, dd, dm, NULL, NULL);
    for (int32_t j = 0; j < d; ++j) {
        store_elem(dtype, dx, base + j, dd[j].rn);
        put_check(lo, hi, mag, base + j, dd[j].lo, dd[j].hi, dm[j]);
    }
}

int muse_oracle_qk_norm_rope_bwd(int dtype, const void* q, const void* k, const void* dq_out,
                                 const void* dk_out, int64_t tokens, int32_t hq, int32_t hkv,
                                 int32_t head_dim, const int32_t* pos, float eps,
                                 float query_scale, int use_rope, int upcast_rope, float rope_base,
                                 int round_grads, void* dq, double* dq_lo, double* dq_hi,
                                 double* dq_mag, void* dk, double* dk_lo, double* dk_hi,
                                 double* dk_mag) {
    if (!valid_dtype(dtype) || tokens < 0 || hq <= 0 || hkv <= 0 || head_dim <= 0 ||
        (head_dim & 1))
        return -1;
    if (tokens && (!q || !k || !dq_out || !dk_out || !dq || !dk || (use_rope && !pos))) return -1;
    float* inv_freq = (float*)malloc(sizeof(float) * (size_t)(head_dim / 2));
    double* xv = (double*)malloc(sizeof(double) * (size_t)head_dim * 3);
    ival* gr = (ival*)malloc(sizeof(ival) * (size_t)head_dim * 2);
    if (!inv_freq || !xv || !gr) { free(inv_freq); free(xv); free(gr); return -1; }
    if (use_rope && muse_oracle_inv_freq(head_dim, rope_base, inv_freq) != 0) {
        free(inv_freq); free(xv); free(gr); return -1;
    }
    double* one = xv + head_dim;
    double* dm = xv + 2 * (int64_t)head_dim;
    ival* dd = gr + head_dim;
    for (int32_t j = 0; j < head_dim; ++j) one[j] = 1.0;
    /* v2 applies to bf16 tensors (FP32 tensors rotate in FP32 in both modes);
     * the exact derivative (round_grads = 0) is the legacy one */
    const int v2 = use_rope && !upcast_rope && dtype == DT_BF16 && round_grads;
    for (int64_t t = 0; t < tokens; ++t) {
        const int32_t p = use_rope ? pos[t] : 0;
        for (int32_t h = 0; h < hq; ++h)
            qk_head_bwd(dtype, q, dq_out, (t * hq + h) * (int64_t)head_dim, head_dim, inv_freq, p,
                        use_rope, v2, eps, 1, query_scale, round_grads, xv, one, gr, dd, dm, dq,
                        dq_lo, dq_hi, dq_mag);
        for (int32_t h = 0; h < hkv; ++h)
            qk_head_bwd(dtype, k, dk_out, (t * hkv + h) * (int64_t)head_dim, head_dim, inv_freq,
                        p, use_rope, v2, eps, 0, 1.0f, round_grads, xv, one, gr, dd, dm, dk, dk_lo,
                        dk_hi, dk_mag);
    }
    free(inv_freq);
    free(xv);
    free(gr);
    return 0;
}

/* ------------------------------------------------------- vision 2-D RoPE */

/* _rope_frequencies (vision page): the table [grid_h * grid_w, D/2, 2] of one
 * row-major patch grid, the (cos, sin) of each adjacent pair's angle.
 * Reading (the page gives the shape only): the first D/4 pairs take the
 * patch's row index h, the other D/4 its column index w, each with the
 * frequencies theta^(-2j/(D/2)), j = 0 .. D/4 - 1 (the text model's inverse
 * frequencies over half the head); the angle is f32(f32(coord) * freq) and
 * its cosine and sine are rounded to FP32.  head_dim a multiple of 4. */
int muse_oracle_vision_rope_frequencies(int32_t head_dim, int32_t grid_h, int32_t grid_w,
                                        float theta, float* out) {
    if (head_dim <= 0 || (head_dim & 3) || grid_h < 0 || grid_w < 0 || !(theta > 0.0f)) return -1;
    if ((int64_t)grid_h * grid_w > 0 && !out) return -1;
    const int32_t quarter = head_dim / 4;
    float* f = (float*)malloc(sizeof(float) * (size_t)quarter);
    if (!f) return -1;
    if (muse_oracle_inv_freq(head_dim / 2, theta, f) != 0) { free(f); return -1; }
    for (int32_t h = 0; h < grid_h; ++h)
        for (int32_t w = 0; w < grid_w; ++w) {
            float* row = out + ((int64_t)h * grid_w + w) * head_dim;
            for (int32_t i = 0; i < head_dim / 2; ++i) {
                const float coord = (float)(i < quarter ? h : w);
                const float phi = coord * f[i < quarter ? i : i - quarter];
                row[2 * i] = (float)cos((double)phi);
                row[2 * i + 1] = (float)sin((double)phi);
            }
        }
    free(f);
    return 0;
}

/* _apply_vision_rope (vision page): adjacent-pair RoPE of q [tokens, hq, D]
 * and k [tokens, hk, D] with the caller's table freqs [tokens, D/2, 2] of
 * (cos, sin) per token and pair: y[2i] = a c - b s, y[2i+1] = a s + b c, in
 * FP32 arithmetic on the Q/K values, cast once to their dtype (reading: the
 * legacy precision of the text rotation). */
static void vision_rope_rows(int dtype, const void* x, int64_t tokens, int32_t heads, int32_t d,
                             const float* freqs, void* out, double* lo, double* hi, double* mag) {
    for (int64_t t = 0; t < tokens; ++t)
        for (int32_t h = 0; h < heads; ++h) {
            const int64_t base = (t * heads + h) * (int64_t)d;
            for (int32_t i = 0; i < d / 2; ++i) {
                const double c = (double)freqs[(t * (d / 2) + i) * 2];
                const double s = (double)freqs[(t * (d / 2) + i) * 2 + 1];
                const double a = load_elem(dtype, x, base + 2 * i);
                const double b = load_elem(dtype, x, base + 2 * i + 1);
                const double y0 = a * c - b * s, y1 = a * s + b * c;
                store_elem(dtype, out, base + 2 * i, y0);
                store_elem(dtype, out, base + 2 * i + 1, y1);
                put_check(lo, hi, mag, base + 2 * i, y0, y0, fabs(a * c) + fabs(b * s));
                put_check(lo, hi, mag, base + 2 * i + 1, y1, y1, fabs(a * s) + fabs(b * c));
            }
        }
}

int muse_oracle_vision_rope(int dtype, const void* q, const void* k, int64_t tokens, int32_t hq,
                            int32_t hk, int32_t head_dim, const float* freqs, void* q_out,
                            double* q_lo, double* q_hi, double* q_mag, void* k_out, double* k_lo,
                            double* k_hi, double* k_mag) {
    if (!valid_dtype(dtype) || tokens < 0 || hq <= 0 || hk <= 0 || head_dim <= 0 || (head_dim & 1))
        return -1;
    if (tokens && (!q || !k || !freqs || !q_out || !k_out)) return -1;
    vision_rope_rows(dtype, q, tokens, hq, head_dim, freqs, q_out, q_lo, q_hi, q_mag);
    vision_rope_rows(dtype, k, tokens, hk, head_dim, freqs, k_out, k_lo, k_hi, k_mag);
    return 0;
}
