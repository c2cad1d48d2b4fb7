/*
 * mla_oracle.c -- plain fp64 CPU oracle for Multi-head Latent Attention decode,
 * in both the absorbed (MQA) mode and the naive (MHA) mode.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg may load this library.  It shares no code, header, table or
 * helper with the CUDA library; it is deliberately slow and written to be
 * checked against the pages by eye: no blocking, no fusion, no reordering
 * beyond what each definition states.  Parallelism (OpenMP) is only over
 * independent (query, head) pairs.
 *
 * Where the method comes from (itwiki article "멀티 헤드 잠재 어텐션",
 * i.e. "Multi-head latent attention"):
 *   - section 구조 / 키·값 공동 압축 (structure, joint KV compression):
 *       c^KV_t = W^DKV h_t,  k^C_t = W^UK c^KV_t,  v^C_t = W^UV c^KV_t,
 *       W^UK, W^UV in R^{n_h d_h x d_c}; only c^KV_t is cached.
 *   - section 행렬 흡수 (matrix absorption): the score q^T W^UK c equals
 *       (W^UK^T q)^T c, so the query is moved into the latent space; the value
 *       side multiplies W^UV after the weighted sum over c^KV.
 *   - section 분리 RoPE (decoupled RoPE): q_{t,i} = [q^C_{t,i}; q^R_{t,i}],
 *       k_{j,i} = [k^C_{j,i}; k^R_j] with one k^R shared by all heads, and
 *       o_{t,i} = sum_{j<=t} softmax_j(q_{t,i}^T k_{j,i} / sqrt(d_h + d_h^R)) v^C_{j,i}.
 *   - section 구현 (implementation): half-split RoPE with base 1e4 whose angle for
 *       pair k is pos * base^(-2k/d_R); the MHA-mode and MQA-mode forwards.
 * The MHA lecture page "MHA · GQA · MQA · MLA", section "Why Projection
 * Absorption Helps", states the same identity q^T W_UK c = (W_UK^T q)^T c.
 *
 * FP8 content cache: the QuantMLA review page, section "Motivation & Problem
 * Statement", describes an FP8 content cache next to a bf16 RoPE-key cache.  The
 * pages fix no scale granularity or rounding; this oracle reads it as one fp32
 * scale per token, s = amax/448 (s = 1 when amax = 0), codes = e4m3 of c/s with
 * round-to-nearest-even and saturation to +-448.  The e4m3 code definition
 * (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent 0 is
 * subnormal; S.1111.111 is NaN; no infinities) is the OCP 8-bit floating point
 * format.
 *
 * Parity pins for every function here live in tests/test_oracle_pins.py.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* RoPE (구현 section: half-split pairing, angle pos * base^(-2k/d_R)).       */
/* ------------------------------------------------------------------------- */

/* out = RoPE(x, pos).  Pair k (k < d_r/2) is (x[k], x[k + d_r/2]); it is rotated
 * by theta_k = pos * base^(-2k/d_r):
 *   out[k]          = x[k] cos theta_k - x[k + d_r/2] sin theta_k
 *   out[k + d_r/2]  = x[k + d_r/2] cos theta_k + x[k] sin theta_k
 * `x` and `out` must not overlap. */
void mla_oracle_rope(int d_r, double base, double pos, const double *x, double *out)
{
    int half = d_r / 2;
    for (int k = 0; k < half; ++k) {
        double inv_freq = 1.0 / pow(base, (double)(2 * k) / (double)d_r);
        double theta = pos * inv_freq;
        double c = cos(theta), s = sin(theta);
        out[k] = x[k] * c - x[k + half] * s;
        out[k + half] = x[k + half] * c + x[k] * s;
    }
}

/* ------------------------------------------------------------------------- */
/* Softmax (분리 RoPE section, output equation).                              */
/* ------------------------------------------------------------------------- */

/* p[j] = exp(s[j]) / sum_k exp(s[k]) over j < n, computed with the maximum
 * subtracted first (two passes).  Returns the natural-log normaliser
 * lse = log(sum_j exp(s[j])).  n must be >= 1. */
double mla_oracle_softmax(int n, const double *s, double *p)
{
    double m = s[0];
    for (int j = 1; j < n; ++j)
        if (s[j] > m) m = s[j];
    double z = 0.0;
    for (int j = 0; j < n; ++j) {
        p[j] = exp(s[j] - m);
        z += p[j];
    }
    for (int j = 0; j < n; ++j) p[j] /= z;
    return m + log(z);
}

/* ------------------------------------------------------------------------- */
/* Absorbed (MQA) mode, step by step, in the order of the 구현 section's       */
/* forward_absorbed and the 행렬 흡수 section.                                 */
/* ------------------------------------------------------------------------- */

/* q_lat = W^UK_h^T q_c: the query of head h moved into the d_c latent space.
 * w_uk is the [n_h*d_h, d_c] row-major weight; head h owns rows h*d_h .. h*d_h+d_h-1. */
void mla_oracle_absorb_query(int d_h, int d_c, int h, const double *w_uk,
                             const double *q_c, double *q_lat)
{
    for (int c = 0; c < d_c; ++c) {
        double acc = 0.0;
        for (int k = 0; k < d_h; ++k)
            acc += w_uk[((size_t)h * d_h + k) * d_c + c] * q_c[k];
        q_lat[c] = acc;
    }
}

/* Value up-projection of head h: o = W^UV_h x  (d_h <- d_c). */
void mla_oracle_up_project(int d_h, int d_c, int h, const double *w, const double *x,
                           double *o)
{
    for (int d = 0; d < d_h; ++d) {
        double acc = 0.0;
        for (int c = 0; c < d_c; ++c)
            acc += w[((size_t)h * d_h + d) * d_c + c] * x[c];
        o[d] = acc;
    }
}

static double dot(int n, const double *a, const double *b)
{
    double acc = 0.0;
    for (int k = 0; k < n; ++k) acc += a[k] * b[k];
    return acc;
}

/* Inputs of one batched decode call (both modes).
 *   B sequences, s_q queries per sequence (T = B*s_q query tokens).
 *   q_c   [T, n_h, d_h]   content query q^C
 *   q_r   [T, n_h, d_r]   RoPE query BEFORE rotation (W^QR c^Q)
 *   q_pos [T]             position of each query token
 *   ctx_off [B+1]         sequence b owns cached tokens ctx_off[b] .. ctx_off[b+1]-1
 *   c_kv  [sum L, d_c]    cached latent c^KV; token j of sequence b sits at position j
 *   k_r   [sum L, d_r]    RoPE key BEFORE rotation (W^KR h), rotated here by position j
 *   w_uk, w_uv [n_h*d_h, d_c]
 * Query t attends to its sequence's tokens j with j <= q_pos[t]. */
typedef struct {
    int B, s_q, n_h, d_h, d_c, d_r;
    double rope_base;
    const double *q_c, *q_r;
    const int64_t *q_pos, *ctx_off;
    const double *c_kv, *k_r, *w_uk, *w_uv;
} oracle_problem;

static int visible_tokens(const oracle_problem *P, int t)
{
    int b = t / P->s_q;
    int64_t L = P->ctx_off[b + 1] - P->ctx_off[b];
    int64_t n = P->q_pos[t] + 1;
    return (int)(n < L ? n : L);
}

/* RoPE of every cached key (k^R_j = RoPE(W^KR h_j) at position j). */
static double *rotate_all_keys(const oracle_problem *P)
{
    int64_t total = P->ctx_off[P->B];
    double *kr = (double *)malloc(sizeof(double) * (size_t)(total > 0 ? total : 1) * P->d_r);
    for (int b = 0; b < P->B; ++b)
        for (int64_t j = P->ctx_off[b]; j < P->ctx_off[b + 1]; ++j)
            mla_oracle_rope(P->d_r, P->rope_base, (double)(j - P->ctx_off[b]),
                            P->k_r + (size_t)j * P->d_r, kr + (size_t)j * P->d_r);
    return kr;
}

/* Absorbed mode for the whole batch.  Outputs (each may be NULL):
 *   q_lat [T, n_h, d_c], o_lat [T, n_h, d_c], lse [T, n_h], o [T, n_h, d_h],
 *   probs [T, n_h, probs_stride] (softmax weights of the visible tokens). */
int mla_oracle_decode_absorbed(int B, int s_q, int n_h, int d_h, int d_c, int d_r,
                               double rope_base, const double *q_c, const double *q_r,
                               const int64_t *q_pos, const int64_t *ctx_off,
                               const double *c_kv, const double *k_r,
                               const double *w_uk, const double *w_uv,
                               double *q_lat_out, double *o_lat_out, double *lse_out,
                               double *o_out, double *probs_out, int probs_stride)
{
    oracle_problem P = {B, s_q, n_h, d_h, d_c, d_r, rope_base, q_c, q_r,
                        q_pos, ctx_off, c_kv, k_r, w_uk, w_uv};
    if (B < 0 || s_q < 1 || n_h < 1 || d_h < 1 || d_c < 1 || d_r < 2 || (d_r & 1)) return 1;
    for (int b = 0; b < B; ++b)
        if (ctx_off[b + 1] - ctx_off[b] < 1) return 2;
    double *kr = rotate_all_keys(&P);
    const double scale = 1.0 / sqrt((double)(d_h + d_r));
    const int T = B * s_q;
    int err = 0;

#pragma omp parallel for schedule(dynamic, 1)
    for (int th = 0; th < T * n_h; ++th) {
        int t = th / n_h, h = th % n_h;
        int b = t / s_q;
        const double *c_seq = c_kv + (size_t)ctx_off[b] * d_c;
        const double *kr_seq = kr + (size_t)ctx_off[b] * d_r;
        int n = visible_tokens(&P, t);
        if (n < 1) { err = 3; continue; }
        double *q_lat = (double *)malloc(sizeof(double) * d_c);
        double *q_rot = (double *)malloc(sizeof(double) * d_r);
        double *s = (double *)malloc(sizeof(double) * n);
        double *p = (double *)malloc(sizeof(double) * n);
        double *o_lat = (double *)malloc(sizeof(double) * d_c);

        /* q_lat = W^UK_h^T q^C (행렬 흡수); q^R rotated at the query's position. */
        mla_oracle_absorb_query(d_h, d_c, h, w_uk, q_c + ((size_t)t * n_h + h) * d_h, q_lat);
        mla_oracle_rope(d_r, rope_base, (double)q_pos[t], q_r + ((size_t)t * n_h + h) * d_r,
                        q_rot);
        /* s_j = (q_lat . c_j + q^R . k^R_j) / sqrt(d_h + d_R) over the (d_c + d_R)-wide row. */
        for (int j = 0; j < n; ++j)
            s[j] = (dot(d_c, q_lat, c_seq + (size_t)j * d_c) +
                    dot(d_r, q_rot, kr_seq + (size_t)j * d_r)) * scale;
        double lse = mla_oracle_softmax(n, s, p);
        /* o_lat = sum_j p_j c_j: every head aggregates the same c^KV. */
        for (int c = 0; c < d_c; ++c) {
            double acc = 0.0;
            for (int j = 0; j < n; ++j) acc += p[j] * c_seq[(size_t)j * d_c + c];
            o_lat[c] = acc;
        }
        size_t row = (size_t)t * n_h + h;
        if (q_lat_out) memcpy(q_lat_out + row * d_c, q_lat, sizeof(double) * d_c);
        if (o_lat_out) memcpy(o_lat_out + row * d_c, o_lat, sizeof(double) * d_c);
        if (lse_out) lse_out[row] = lse;
        /* o = W^UV_h o_lat: the value up-projection applied after aggregation. */
        if (o_out) mla_oracle_up_project(d_h, d_c, h, w_uv, o_lat, o_out + row * d_h);
        if (probs_out) {
            for (int j = 0; j < probs_stride; ++j)
                probs_out[row * probs_stride + j] = j < n ? p[j] : 0.0;
        }
        free(q_lat); free(q_rot); free(s); free(p); free(o_lat);
    }
    free(kr);
    return err;
}

/* Naive (MHA) mode for the whole batch: the keys and values of every cached
 * token are reconstructed per head, k^C_{j,h} = W^UK_h c_j and v_{j,h} = W^UV_h c_j
 * (구조 section), and attention runs in the d_h-wide head space.
 * Outputs: lse [T, n_h], o [T, n_h, d_h] (each may be NULL). */
int mla_oracle_decode_naive(int B, int s_q, int n_h, int d_h, int d_c, int d_r,
                            double rope_base, const double *q_c, const double *q_r,
                            const int64_t *q_pos, const int64_t *ctx_off,
                            const double *c_kv, const double *k_r,
                            const double *w_uk, const double *w_uv,
                            double *lse_out, double *o_out)
{
    oracle_problem P = {B, s_q, n_h, d_h, d_c, d_r, rope_base, q_c, q_r,
                        q_pos, ctx_off, c_kv, k_r, w_uk, w_uv};
    if (B < 0 || s_q < 1 || n_h < 1 || d_h < 1 || d_c < 1 || d_r < 2 || (d_r & 1)) return 1;
    for (int b = 0; b < B; ++b)
        if (ctx_off[b + 1] - ctx_off[b] < 1) return 2;
    double *kr = rotate_all_keys(&P);
    const double scale = 1.0 / sqrt((double)(d_h + d_r));
    const int T = B * s_q;
    int err = 0;

#pragma omp parallel for schedule(dynamic, 1)
    for (int th = 0; th < T * n_h; ++th) {
        int t = th / n_h, h = th % n_h;
        int b = t / s_q;
        const double *c_seq = c_kv + (size_t)ctx_off[b] * d_c;
        const double *kr_seq = kr + (size_t)ctx_off[b] * d_r;
        int n = visible_tokens(&P, t);
        if (n < 1) { err = 3; continue; }
        double *k_c = (double *)malloc(sizeof(double) * (size_t)n * d_h);
        double *v = (double *)malloc(sizeof(double) * (size_t)n * d_h);
        double *q_rot = (double *)malloc(sizeof(double) * d_r);
        double *s = (double *)malloc(sizeof(double) * n);
        double *p = (double *)malloc(sizeof(double) * n);
        for (int j = 0; j < n; ++j) {
            mla_oracle_up_project(d_h, d_c, h, w_uk, c_seq + (size_t)j * d_c, k_c + (size_t)j * d_h);
            mla_oracle_up_project(d_h, d_c, h, w_uv, c_seq + (size_t)j * d_c, v + (size_t)j * d_h);
        }
        const double *qc = q_c + ((size_t)t * n_h + h) * d_h;
        mla_oracle_rope(d_r, rope_base, (double)q_pos[t], q_r + ((size_t)t * n_h + h) * d_r, q_rot);
        for (int j = 0; j < n; ++j)
            s[j] = (dot(d_h, qc, k_c + (size_t)j * d_h) +
                    dot(d_r, q_rot, kr_seq + (size_t)j * d_r)) * scale;
        double lse = mla_oracle_softmax(n, s, p);
        size_t row = (size_t)t * n_h + h;
        if (lse_out) lse_out[row] = lse;
        if (o_out) {
            for (int d = 0; d < d_h; ++d) {
                double acc = 0.0;
                for (int j = 0; j < n; ++j) acc += p[j] * v[(size_t)j * d_h + d];
                o_out[row * d_h + d] = acc;
            }
        }
        free(k_c); free(v); free(q_rot); free(s); free(p);
    }
    free(kr);
    return err;
}

/* ------------------------------------------------------------------------- */
/* FP8 e4m3 content cache (QuantMLA review, Motivation & Problem Statement;    */
/* code format from the OCP 8-bit floating point definition).                 */
/* ------------------------------------------------------------------------- */

/* Real value of an e4m3 code.  NaN for S.1111.111. */
double mla_oracle_e4m3_value(uint8_t code)
{
    int sign = code >> 7;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    if (e == 0xF && m == 0x7) return NAN;
    double mag = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* e4m3 code of v: round to nearest, ties to the code with an even mantissa,
 * magnitudes beyond 448 saturate to 448.  Found by comparing |v| with every
 * finite non-negative code (0x00 .. 0x7E); NaN maps to 0x7F. */
uint8_t mla_oracle_e4m3_quantize(float v)
{
    if (isnan(v)) return 0x7F;
    double a = fabs((double)v);
    int best = 0;
    double best_err = INFINITY;
    for (int code = 0; code <= 0x7E; ++code) {
        double err = fabs(mla_oracle_e4m3_value((uint8_t)code) - a);
        if (err < best_err || (err == best_err && (code & 1) == 0)) {
            best = code;
            best_err = err;
        }
    }
    return (uint8_t)((signbit(v) ? 0x80 : 0x00) | best);
}

/* Per-token quantisation of one c^KV row of width d_c (fp32 arithmetic, as the
 * row is stored): amax = max |c|, s = amax/448 (at least FLT_MIN; 1 if amax = 0),
 * codes[k] = e4m3(c[k] / s). */
void mla_oracle_quantize_row(int d_c, const float *c, uint8_t *codes, float *scale)
{
    float amax = 0.0f;
    for (int k = 0; k < d_c; ++k) {
        float a = fabsf(c[k]);
        if (a > amax) amax = a;
    }
    float s = 1.0f;
    if (amax > 0.0f) {
        volatile float q = amax / 448.0f; /* fp32 division, rounded once */
        s = q > FLT_MIN ? q : FLT_MIN;
    }
    for (int k = 0; k < d_c; ++k) {
        volatile float x = c[k] / s;
        codes[k] = mla_oracle_e4m3_quantize(x);
    }
    *scale = s;
}

/* Batched form: n rows. */
void mla_oracle_quantize_rows(int64_t n, int d_c, const float *c, uint8_t *codes, float *scales)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        mla_oracle_quantize_row(d_c, c + (size_t)i * d_c, codes + (size_t)i * d_c, scales + i);
}

/* Dequantised row: out[k] = e4m3_value(codes[k]) * scale, in fp64. */
void mla_oracle_dequantize_rows(int64_t n, int d_c, const uint8_t *codes, const float *scales,
                                double *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        for (int k = 0; k < d_c; ++k)
            out[(size_t)i * d_c + k] =
                mla_oracle_e4m3_value(codes[(size_t)i * d_c + k]) * (double)scales[i];
}

/* Number of cached elements per token and layer in the latent cache: the
 * 분리 RoPE section caches c^KV_t and k^R_t together, d_c + d_R elements. */
int mla_oracle_cache_row_elems(int d_c, int d_r) { return d_c + d_r; }

int mla_oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Host threads for the following calls (the results do not depend on it: every (query, head)
 * pair is computed by one thread in a fixed order).  For timing the oracle single-threaded. */
void mla_oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
