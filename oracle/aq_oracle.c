/*
 * CPU oracle for additive-quantised matrix products.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link or
 * call this file: only tests/, __graft_entry__.smoke() and the CPU-baseline /
 * reference arm of bench.py use it.  It shares no code, header, table or
 * constant with the CUDA library; it is written from the method's definition
 * and is deliberately plain and slow (no blocking, no reordering).
 *
 * Sources (web pages on "Extreme Compression of Large Language Models via
 * Additive Quantization", Egiazarian et al., ICML 2024):
 *   - AQLM wiki entry (brain.gartu.xyz), section "Niveau intermédiaire":
 *     each group of weights is approximated by the sum of one vector from each
 *     of K codebooks, w ~ C_1[i_1] + ... + C_K[i_K]; bit rate per weight is
 *     K * log2(codebook size) / group size.
 *   - devtrends.ru summary ("AQLM — Сжимаем языковые модели без потерь"), section "Как это работает технически?":
 *     groups are 8 consecutive weights (in_group_size = 8).
 *   - arXiv 2401.06118 abstract: the GPU/CPU kernels compute the product of
 *     the quantised matrix with activations for token generation.
 * The per-row scale s and the packed code layout are this library's interface
 * (the pages mention neither); the oracle follows their written definitions:
 *   y[o][b] = s[o] * sum_i W[o][i] * x[i][b],
 *   W[o][8g+j] = RN16( sum_k C_k[codes[o][g][k]][j] ).
 *
 * Readings of points the pages leave open:
 *   - the sum over k is formed exactly (fp64 holds any sum of <= 8 binary16
 *     values exactly) and rounded once to binary16, ties to even;
 *   - the product with x and the scale are taken in fp64 from the binary16
 *     values, no intermediate rounding;
 *   - codes are unsigned, code k selects a row of codebook k;
 *   - for the gradient with respect to the codebooks and scales (the fine-
 *     tuning step the wiki entry describes: codebooks are learned jointly
 *     with the codes), the decode's rounding is taken as the identity.
 *
 * Pins (tests/test_oracle_pins.py): conversions against numpy's binary16,
 * exhaustive single-group decode, one-hot codebooks, additivity, permutation
 * invariance, integer-exact products, pure-Python brute force on tiny inputs,
 * the pages' bit-rate examples and model sizes, pack round trip and
 * hand-worked layout offsets.  tests/test_oracle_mutants.py checks the pins
 * themselves: copies of this file with one planted slip each must fail them.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define AQO_GROUP 8

/* ------------------------------------------------------------------------ */
/* IEEE 754 binary16, written from the format definition:                   */
/* 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.                 */
/* ------------------------------------------------------------------------ */

double aqo_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -24); /* zero or subnormal: f * 2^-24 */
    } else if (e == 31) {
        v = f ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + f), e - 25); /* 1.f * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* q >= 0 holds an exact value; return it rounded to an integer, ties to even. */
static double round_half_even(double q)
{
    double fl = floor(q);
    double d = q - fl; /* exact: q and fl share the exponent range */
    if (d > 0.5) return fl + 1.0;
    if (d < 0.5) return fl;
    return (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
}

uint16_t aqo_double_to_half(double v)
{
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (isnan(v)) return (uint16_t)(sign | 0x7e00);
    /* 65504 is the largest finite value; the midpoint to 2^16 is 65520,
     * which rounds to even (upwards, to infinity). */
    if (a >= 65520.0) return (uint16_t)(sign | 0x7c00);
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: value = m * 2^-24, m in [0, 1024]; m == 1024 is
         * the smallest normal number and encodes correctly as 0x0400. */
        double m = round_half_even(ldexp(a, 24));
        return (uint16_t)(sign | (uint16_t)m);
    }
    int ex;
    frexp(a, &ex); /* a = f * 2^ex, f in [0.5, 1) -> a in [2^(ex-1), 2^ex) */
    int e = ex - 1;                             /* unbiased exponent */
    double m = round_half_even(ldexp(a, 10 - e)); /* in [1024, 2048] */
    if (m == 2048.0) {
        m = 1024.0;
        e += 1;
    }
    if (e + 15 >= 31) return (uint16_t)(sign | 0x7c00);
    return (uint16_t)(sign | (uint16_t)((e + 15) << 10) | (uint16_t)(m - 1024.0));
}

/* ------------------------------------------------------------------------ */
/* Bit rate and storage (wiki entry, "Niveau intermédiaire").               */
/* ------------------------------------------------------------------------ */

/* bits per weight = K * log2(codebook size) / group size; codebook size 2^B */
double aqo_bits_per_weight(int K, int B, int g)
{
    return (double)K * (double)B / (double)g;
}

/* Bytes one quantised layer occupies: codes at K*B bits per group of 8,
 * K codebooks of 2^B binary16 8-vectors, one binary16 scale per row. */
double aqo_layer_bytes(int64_t out, int64_t in, int K, int B)
{
    double code_bits = (double)out * (double)(in / AQO_GROUP) * K * B;
    double codebook_bytes = (double)K * ldexp(1.0, B) * AQO_GROUP * 2.0;
    return code_bits / 8.0 + codebook_bytes + 2.0 * (double)out;
}

/* ------------------------------------------------------------------------ */
/* Decode (additive reconstruction of one group).                           */
/* ------------------------------------------------------------------------ */

static uint32_t code_at(const void *codes, int B, int64_t idx)
{
    if (B <= 8) return ((const uint8_t *)codes)[idx];
    return ((const uint16_t *)codes)[idx];
}

static int check_scheme(int64_t out, int64_t in, int K, int B)
{
    if (out < 0 || in < 0 || in % AQO_GROUP) return -1;
    if (K < 1 || K > 8 || B < 1 || B > 16) return -1;
    return 0;
}

/* Row o of W as doubles (each value already rounded to binary16). */
static void decode_row(int64_t o, int64_t in, int K, int B, const void *codes,
                       const uint16_t *codebooks, double *row)
{
    int64_t G = in / AQO_GROUP;
    int64_t ncw = (int64_t)1 << B;
    for (int64_t g = 0; g < G; ++g) {
        for (int j = 0; j < AQO_GROUP; ++j) {
            /* The sum starts from the first term (not from +0), so a lone
             * -0 codeword entry stays -0; it is exact: <= 8 binary16 terms. */
            double sum = 0.0;
            for (int k = 0; k < K; ++k) {
                uint32_t c = code_at(codes, B, (o * G + g) * K + k);
                double term = aqo_half_to_double(codebooks[((int64_t)k * ncw + c) * AQO_GROUP + j]);
                sum = (k == 0) ? term : sum + term;
            }
            row[g * AQO_GROUP + j] = aqo_half_to_double(aqo_double_to_half(sum));
        }
    }
}

/* W[o][i] as binary16 bits; with scales != NULL, RN16(s[o] * W[o][i]). */
int aqo_decode(int64_t out, int64_t in, int K, int B, const void *codes,
               const uint16_t *codebooks, const uint16_t *scales, uint16_t *w)
{
    if (check_scheme(out, in, K, B)) return -1;
    double *row = (double *)malloc(sizeof(double) * (size_t)(in > 0 ? in : 1));
    if (!row) return -2;
    for (int64_t o = 0; o < out; ++o) {
        decode_row(o, in, K, B, codes, codebooks, row);
        double s = scales ? aqo_half_to_double(scales[o]) : 1.0;
        for (int64_t i = 0; i < in; ++i)
            w[o * in + i] = scales ? aqo_double_to_half(s * row[i])
                                   : aqo_double_to_half(row[i]);
    }
    free(row);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Product y = diag(s) * W * x in fp64 (x is [in][n]).                      */
/* rows == NULL: all rows, y is [out][n]; else y is [nrows][n] for the      */
/* listed rows.  bound (optional) receives sum_i |s||W||x| per element, the */
/* scale of the tolerance the GPU results are checked against.             */
/* ------------------------------------------------------------------------ */

int aqo_matmul(int64_t out, int64_t in, int K, int B, const void *codes,
               const uint16_t *codebooks, const uint16_t *scales,
               const uint16_t *x, int64_t n, const int64_t *rows, int64_t nrows,
               double *y, double *bound, int threads)
{
    if (check_scheme(out, in, K, B) || n < 0) return -1;
    if (!rows) nrows = out;
    for (int64_t r = 0; rows && r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= out) return -1;
    double *xd = (double *)malloc(sizeof(double) * (size_t)(in * n > 0 ? in * n : 1));
    if (!xd) return -2;
    for (int64_t t = 0; t < in * n; ++t) xd[t] = aqo_half_to_double(x[t]);
    int err = 0;
#ifdef _OPENMP
    if (threads < 1) threads = 1;
#pragma omp parallel num_threads(threads)
#endif
    {
        double *row = (double *)malloc(sizeof(double) * (size_t)(in > 0 ? in : 1));
        if (!row) {
            err = -2;
        } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 8)
#endif
            for (int64_t r = 0; r < nrows; ++r) {
                int64_t o = rows ? rows[r] : r;
                decode_row(o, in, K, B, codes, codebooks, row);
                double s = scales ? aqo_half_to_double(scales[o]) : 1.0;
                for (int64_t b = 0; b < n; ++b) {
                    double acc = 0.0, mag = 0.0;
                    for (int64_t i = 0; i < in; ++i) {
                        acc += row[i] * xd[i * n + b];
                        mag += fabs(row[i] * xd[i * n + b]);
                    }
                    y[r * n + b] = s * acc;
                    if (bound) bound[r * n + b] = fabs(s) * mag;
                }
            }
            free(row);
        }
    }
    free(xd);
    return err;
}

/* ------------------------------------------------------------------------ */
/* Gradient with respect to the row scales and the codebooks.               */
/*                                                                          */
/* For L = sum_{o,b} gy[o][b] y[o][b] with y = diag(s) W x and              */
/* W[o][8g+j] = RN16(sum_k C_k[i_k][j]) (AQLM wiki entry, "Niveau            */
/* intermédiaire": the additive decode), the rounding is taken as the       */
/* identity (its derivative wherever it is differentiable), so each weight  */
/* depends on codeword entry C_k[c][j] with derivative 1 when i_k = c:       */
/*   M[o][i]         = sum_b gy[o][b] x[i][b]                               */
/*   grad_s[o]       = sum_i W[o][i] M[o][i]                                */
/*   grad_C[k][c][j] = sum of s[o] M[o][8g+j] over every (o, g) whose code   */
/*                     k is c                                               */
/* with the magnitudes of the same sums (absolute value of every term) as   */
/* error bounds.  All in double from the binary16 inputs.                   */
/* ------------------------------------------------------------------------ */

int aqo_backward(int64_t out, int64_t in, int K, int B, const void *codes,
                 const uint16_t *codebooks, const uint16_t *scales, const uint16_t *x,
                 const uint16_t *gy, int64_t n, double *grad_s, double *grad_s_bound,
                 double *grad_cb, double *grad_cb_bound)
{
    if (check_scheme(out, in, K, B) || n < 0) return -1;
    int64_t G = in / AQO_GROUP;
    int64_t ncb = (int64_t)K << B;
    double *xd = (double *)malloc(sizeof(double) * (size_t)(in * n > 0 ? in * n : 1));
    double *row = (double *)malloc(sizeof(double) * (size_t)(in > 0 ? in : 1));
    double *m = (double *)malloc(sizeof(double) * (size_t)(in > 0 ? in : 1));
    double *mabs = (double *)malloc(sizeof(double) * (size_t)(in > 0 ? in : 1));
    if (!xd || !row || !m || !mabs) {
        free(xd); free(row); free(m); free(mabs);
        return -2;
    }
    for (int64_t t = 0; t < in * n; ++t) xd[t] = aqo_half_to_double(x[t]);
    for (int64_t e = 0; e < ncb * AQO_GROUP; ++e) {
        if (grad_cb) grad_cb[e] = 0.0;
        if (grad_cb_bound) grad_cb_bound[e] = 0.0;
    }
    for (int64_t o = 0; o < out; ++o) {
        decode_row(o, in, K, B, codes, codebooks, row);
        double s = scales ? aqo_half_to_double(scales[o]) : 1.0;
        for (int64_t i = 0; i < in; ++i) {
            double acc = 0.0, mag = 0.0;
            for (int64_t b = 0; b < n; ++b) {
                double t = aqo_half_to_double(gy[o * n + b]) * xd[i * n + b];
                acc += t;
                mag += fabs(t);
            }
            m[i] = acc;
            mabs[i] = mag;
        }
        double gs = 0.0, gsb = 0.0;
        for (int64_t i = 0; i < in; ++i) {
            gs += row[i] * m[i];
            gsb += fabs(row[i]) * mabs[i];
        }
        if (grad_s) grad_s[o] = gs;
        if (grad_s_bound) grad_s_bound[o] = gsb;
        for (int64_t g = 0; g < G; ++g) {
            for (int k = 0; k < K; ++k) {
                uint32_t c = code_at(codes, B, (o * G + g) * K + k);
                int64_t base = (((int64_t)k << B) + c) * AQO_GROUP;
                for (int j = 0; j < AQO_GROUP; ++j) {
                    if (grad_cb) grad_cb[base + j] += s * m[g * AQO_GROUP + j];
                    if (grad_cb_bound) grad_cb_bound[base + j] += fabs(s) * mabs[g * AQO_GROUP + j];
                }
            }
        }
    }
    free(xd); free(row); free(m); free(mabs);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Encoder: beam search of the codes for fixed codebooks.                   */
/*                                                                          */
/* The AQLM wiki entry ("Niveau tech avancé") states the objective          */
/* sum over layers of || W - sum_k C_k[i_k] ||^2_H with H = 2 X^T X from     */
/* calibration activations, and that the codes are assigned by beam search  */
/* rather than greedily.  || (W - What) X^T ||^2 is a sum over output rows   */
/* of e_o^T (X^T X) e_o, so every row is its own problem.  Reading taken:    */
/*   - the reconstruction is the exact sum of the codewords (no rounding);   */
/*   - the beam search runs over the K codes of one group (the "index       */
/*     combination" of that group), the other groups fixed: groups in       */
/*     ascending order, starting from the given codes; for group g the      */
/*     codebooks are visited k = 0..K-1; at each, every beam proposes each   */
/*     of the 2^B codes for slot (g, k); the `beam` proposals with the      */
/*     smallest objective survive, ordered by (objective, parent beam,      */
/*     code) so that ties resolve the same way every time (beams differ in  */
/*     an already visited code of the group, so proposals never repeat);    */
/*   - after the group's last codebook the first surviving beam is kept     */
/*     and the next group starts from it as the only beam.                  */
/* Every proposal is scored by the quadratic form written out, in double.   */
/* ------------------------------------------------------------------------ */

static double quad_form(const double *e, const double *h, int64_t in)
{
    double f = 0.0;
    for (int64_t a = 0; a < in; ++a) {
        double t = 0.0;
        for (int64_t b = 0; b < in; ++b) t += h[a * in + b] * e[b];
        f += e[a] * t;
    }
    return f;
}

/* Row error w - sum_k C_k[codes[g][k]] for one row's codes [G][K]. */
static void row_error(int64_t in, int K, int B, const uint32_t *codes, const double *w,
                      const uint16_t *codebooks, double *e)
{
    int64_t G = in / AQO_GROUP;
    for (int64_t g = 0; g < G; ++g)
        for (int j = 0; j < AQO_GROUP; ++j) {
            double sum = 0.0;
            for (int k = 0; k < K; ++k)
                sum += aqo_half_to_double(codebooks[(((int64_t)k << B) + codes[g * K + k]) * AQO_GROUP + j]);
            e[g * AQO_GROUP + j] = w[g * AQO_GROUP + j] - sum;
        }
}

typedef struct { double f; int parent; uint32_t code; } aqo_prop;

static int prop_less(const aqo_prop *a, const aqo_prop *b)
{
    if (a->f != b->f) return a->f < b->f;
    if (a->parent != b->parent) return a->parent < b->parent;
    return a->code < b->code;
}

/* codes_in / codes_out: [out][in/8][K] as uint32 (any B); w binary16
 * [out][in]; h fp32 [in][in]; objective_out[out] (optional) the final
 * objective of each row. */
int aqo_encode(int64_t out, int64_t in, int K, int B, const uint16_t *w, const float *h,
               const uint16_t *codebooks, const uint32_t *codes_in, int beam,
               uint32_t *codes_out, double *objective_out)
{
    if (check_scheme(out, in, K, B) || beam < 1) return -1;
    int64_t G = in / AQO_GROUP, S = G * K, ncw = (int64_t)1 << B;
    double *hd = (double *)malloc(sizeof(double) * (size_t)(in * in > 0 ? in * in : 1));
    double *wd = (double *)malloc(sizeof(double) * (size_t)(in > 0 ? in : 1));
    double *e = (double *)malloc(sizeof(double) * (size_t)(in > 0 ? in : 1));
    uint32_t *cur = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)(beam * S > 0 ? beam * S : 1));
    uint32_t *nxt = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)(beam * S > 0 ? beam * S : 1));
    double *fcur = (double *)malloc(sizeof(double) * (size_t)beam);
    aqo_prop *props = (aqo_prop *)malloc(sizeof(aqo_prop) * (size_t)(beam * ncw));
    uint32_t *trial = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)(S > 0 ? S : 1));
    if (!hd || !wd || !e || !cur || !nxt || !fcur || !props || !trial) {
        free(hd); free(wd); free(e); free(cur); free(nxt); free(fcur); free(props); free(trial);
        return -2;
    }
    for (int64_t t = 0; t < in * in; ++t) hd[t] = (double)h[t];
    for (int64_t o = 0; o < out; ++o) {
        for (int64_t i = 0; i < in; ++i) wd[i] = aqo_half_to_double(w[o * in + i]);
        int nb = 1;
        for (int64_t t = 0; t < S; ++t) cur[t] = codes_in[o * S + t];
        row_error(in, K, B, cur, wd, codebooks, e);
        fcur[0] = quad_form(e, hd, in);
        for (int64_t sl = 0; sl < S; ++sl) {
            if (sl % K == 0) nb = 1;  /* a new group starts from the best beam */
            int np = 0;
            for (int b = 0; b < nb; ++b)
                for (int64_t c = 0; c < ncw; ++c) {
                    for (int64_t t = 0; t < S; ++t) trial[t] = cur[b * S + t];
                    trial[sl] = (uint32_t)c;
                    row_error(in, K, B, trial, wd, codebooks, e);
                    props[np].f = quad_form(e, hd, in);
                    props[np].parent = b;
                    props[np].code = (uint32_t)c;
                    ++np;
                }
            /* keep the `beam` smallest: selection by repeated minimum */
            int keep = np < beam ? np : beam;
            for (int r = 0; r < keep; ++r) {
                int best = r;
                for (int q = r + 1; q < np; ++q)
                    if (prop_less(&props[q], &props[best])) best = q;
                aqo_prop tmp = props[r]; props[r] = props[best]; props[best] = tmp;
            }
            for (int r = 0; r < keep; ++r) {
                for (int64_t t = 0; t < S; ++t) nxt[r * S + t] = cur[props[r].parent * S + t];
                nxt[r * S + sl] = props[r].code;
                fcur[r] = props[r].f;
            }
            nb = keep;
            uint32_t *sw = cur; cur = nxt; nxt = sw;
        }
        for (int64_t t = 0; t < S; ++t) codes_out[o * S + t] = cur[t];
        if (objective_out) objective_out[o] = fcur[0];
    }
    free(hd); free(wd); free(e); free(cur); free(nxt); free(fcur); free(props); free(trial);
    return 0;
}

/* Objective of given codes per row (same definition), for checks. */
int aqo_objective(int64_t out, int64_t in, int K, int B, const uint16_t *w, const float *h,
                  const uint16_t *codebooks, const uint32_t *codes, double *objective)
{
    if (check_scheme(out, in, K, B)) return -1;
    int64_t S = (in / AQO_GROUP) * K;
    double *hd = (double *)malloc(sizeof(double) * (size_t)(in * in > 0 ? in * in : 1));
    double *wd = (double *)malloc(sizeof(double) * (size_t)(in > 0 ? in : 1));
    double *e = (double *)malloc(sizeof(double) * (size_t)(in > 0 ? in : 1));
    if (!hd || !wd || !e) { free(hd); free(wd); free(e); return -2; }
    for (int64_t t = 0; t < in * in; ++t) hd[t] = (double)h[t];
    for (int64_t o = 0; o < out; ++o) {
        for (int64_t i = 0; i < in; ++i) wd[i] = aqo_half_to_double(w[o * in + i]);
        row_error(in, K, B, codes + o * S, wd, codebooks, e);
        objective[o] = quad_form(e, hd, in);
    }
    free(hd); free(wd); free(e);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Packed code layout (the library's documented interface).                 */
/*                                                                          */
/* Each group (o, g) has one word of W = K*B/8 bytes holding its K codes,   */
/* code k in bits [k*B, (k+1)*B) (1x16: the code; 2x8: c0 | c1 << 8; 1x8:   */
/* one byte; 2x16: c0 | c1 << 16; 8x8: eight bytes, c0 first).  Rows are    */
/* padded to a multiple of 8 and groups to a multiple of 32 with zero words.*/
/* Word (o, g) is stored little-endian at byte                              */
/*   ((o / 8) * (Gp / 32) + g / 32) * 256 W + (g % 32) * 8 W + (o % 8) * W  */
/* where Gp is the padded group count: a 256 W-byte tile holds 8 rows x 32  */
/* groups, each 8 W-byte chunk holds one group for 8 consecutive rows.      */
/* ------------------------------------------------------------------------ */

static int packed_scheme_ok(int K, int B)
{
    return (K == 1 && B == 16) || (K == 2 && B == 8) || (K == 1 && B == 8) ||
           (K == 2 && B == 16) || (K == 8 && B == 8);
}

int64_t aqo_packed_bytes(int64_t out, int64_t in, int K, int B)
{
    if (check_scheme(out, in, K, B) || !packed_scheme_ok(K, B)) return -1;
    int64_t rows = (out + 7) / 8 * 8;
    int64_t gp = (in / AQO_GROUP + 31) / 32 * 32;
    return rows * gp * (K * B / 8);
}

static int64_t packed_offset(int64_t o, int64_t g, int64_t gp, int64_t W)
{
    return ((o / 8) * (gp / 32) + g / 32) * 256 * W + (g % 32) * 8 * W + (o % 8) * W;
}

int aqo_pack(int64_t out, int64_t in, int K, int B, const void *codes, uint8_t *packed)
{
    int64_t nbytes = aqo_packed_bytes(out, in, K, B);
    if (nbytes < 0) return -1;
    int64_t G = in / AQO_GROUP;
    int64_t gp = (G + 31) / 32 * 32;
    int64_t W = K * B / 8;
    memset(packed, 0, (size_t)nbytes);
    for (int64_t o = 0; o < out; ++o) {
        for (int64_t g = 0; g < G; ++g) {
            uint64_t word = 0;
            for (int k = 0; k < K; ++k)
                word |= (uint64_t)code_at(codes, B, (o * G + g) * K + k) << (k * B);
            int64_t at = packed_offset(o, g, gp, W);
            for (int64_t b = 0; b < W; ++b) packed[at + b] = (uint8_t)(word >> (8 * b));
        }
    }
    return 0;
}

int aqo_unpack(int64_t out, int64_t in, int K, int B, const uint8_t *packed, void *codes)
{
    if (aqo_packed_bytes(out, in, K, B) < 0) return -1;
    int64_t G = in / AQO_GROUP;
    int64_t gp = (G + 31) / 32 * 32;
    int64_t W = K * B / 8;
    uint64_t mask = (B == 16) ? 0xffffu : 0xffu;
    for (int64_t o = 0; o < out; ++o) {
        for (int64_t g = 0; g < G; ++g) {
            int64_t at = packed_offset(o, g, gp, W);
            uint64_t word = 0;
            for (int64_t b = 0; b < W; ++b) word |= (uint64_t)packed[at + b] << (8 * b);
            for (int k = 0; k < K; ++k) {
                uint64_t c = (word >> (k * B)) & mask;
                if (B <= 8)
                    ((uint8_t *)codes)[(o * G + g) * K + k] = (uint8_t)c;
                else
                    ((uint16_t *)codes)[(o * G + g) * K + k] = (uint16_t)c;
            }
        }
    }
    return 0;
}

int aqo_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
