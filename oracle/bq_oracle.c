/*
 * bq_oracle.c -- TEST INFRASTRUCTURE ONLY (see bq_oracle.h).
 *
 * The plain CPU definition of the binary / ternary g128 weight path, in FP64.
 * Nothing here is blocked, fused or reordered beyond the definitions it
 * cites.  Where the pages leave a step open, the reading taken is named at the
 * function.  Build: gcc -O2 -std=c11 -ffp-contract=off -fopenmp -fPIC -shared.
 */
#include "bq_oracle.h"

#include <math.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define GROUP 128

/* ------------------------------------------------------------------------ */
/* IEEE-754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
 * Normal: (1 + f/2^10) * 2^(e-15); subnormal (e = 0): f * 2^-24;
 * e = 31: infinity (f = 0) or NaN.                                          */
double bqo_half_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 31;
    int f = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);
    else if (e == 31)
        v = (f == 0) ? INFINITY : NAN;
    else
        v = ldexp((double)(1024 + f), e - 25);
    return sign ? -v : v;
}

/* Round a non-negative integer-valued-or-not quotient n to the nearest
 * integer, ties to even. */
static double round_half_even(double n) {
    double fl = floor(n);
    double d = n - fl;                 /* exact: n and fl share the binade */
    if (d > 0.5) return fl + 1.0;
    if (d < 0.5) return fl;
    return (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
}

/* Generic "round |v| to p significant bits with minimum exponent emin and
 * largest finite exponent emax" used for binary16 (p=11) and bfloat16 (p=8).
 * Returns the rounded magnitude; *overflow set when it exceeds the largest
 * finite value.                                                              */
static double round_to_format(double a, int p, int emin, int emax, int* overflow) {
    *overflow = 0;
    if (a == 0.0) return 0.0;
    int ex;
    frexp(a, &ex);                      /* a = m * 2^ex, m in [0.5, 1) */
    int e = ex - 1;                     /* a in [2^e, 2^(e+1)) */
    if (e < emin) e = emin;             /* subnormal range: fixed quantum */
    double q = ldexp(1.0, e - (p - 1)); /* quantum (one unit in the last place) */
    double r = round_half_even(a / q) * q;
    double maxfinite = ldexp(2.0 - ldexp(1.0, -(p - 1)), emax);
    if (r > maxfinite) *overflow = 1;
    return r;
}

uint16_t bqo_double_to_half(double v) {
    if (isnan(v)) return 0x7E00;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    int of;
    double r = round_to_format(a, 11, -14, 15, &of);
    if (of || isinf(a)) return sign | 0x7C00;
    if (r == 0.0) return sign;
    if (r < ldexp(1.0, -14))                       /* subnormal */
        return sign | (uint16_t)(r / ldexp(1.0, -24));
    int ex;
    double m = frexp(r, &ex);                      /* r = m 2^ex, m in [0.5,1) */
    int e = ex - 1;                                /* r = (2m) 2^e            */
    uint16_t frac = (uint16_t)((2.0 * m - 1.0) * 1024.0);
    return sign | (uint16_t)((e + 15) << 10) | frac;
}

/* bfloat16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits. */
double bqo_bf16_to_double(uint16_t b) {
    int sign = (b >> 15) & 1;
    int e = (b >> 7) & 255;
    int f = b & 127;
    double v;
    if (e == 0)
        v = ldexp((double)f, -133);
    else if (e == 255)
        v = (f == 0) ? INFINITY : NAN;
    else
        v = ldexp((double)(128 + f), e - 134);
    return sign ? -v : v;
}

uint16_t bqo_double_to_bf16(double v) {
    if (isnan(v)) return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    int of;
    double r = round_to_format(a, 8, -126, 127, &of);
    if (of || isinf(a)) return sign | 0x7F80;
    if (r == 0.0) return sign;
    if (r < ldexp(1.0, -126))
        return sign | (uint16_t)(r / ldexp(1.0, -133));
    int ex;
    double m = frexp(r, &ex);
    int e = ex - 1;
    uint16_t frac = (uint16_t)((2.0 * m - 1.0) * 128.0);
    return sign | (uint16_t)((e + 127) << 7) | frac;
}

/* ------------------------------------------------------------------------ */
/* Storage.  [P1] one sign bit per weight + one FP16 scale per 128 weights;
 * [P2]/[P3 §2.4] trits in 2-bit slots; [P3 §2.4] five trits per byte.
 * Reading for 5-per-byte: a 128-trit group is 25 bytes of five trits plus a
 * 26th byte holding the last three trits.                                    */
static int fmt_ok(int fmt) {
    return fmt == BQO_Q1G128 || fmt == BQO_T2G128 || fmt == BQO_T5P8G128;
}

int64_t bqo_codes_bytes(int fmt, int64_t n, int64_t k) {
    if ((!fmt_ok(fmt) && fmt != BQO_A1G128) || n < 0 || k < 0 || k % GROUP) return -1;
    if (fmt == BQO_Q1G128 || fmt == BQO_A1G128) return n * (k / 8);
    if (fmt == BQO_T2G128) return n * (k / 4);
    return n * (k / GROUP) * 26;
}

int64_t bqo_scales_bytes(int64_t n, int64_t k) {
    if (n < 0 || k < 0 || k % GROUP) return -1;
    return n * (k / GROUP) * 2;
}

double bqo_effective_bits(int fmt) {
    if (fmt == BQO_A1G128) /* one bit plus an FP16 (scale, bias) pair per 128 */
        return 8.0 * (double)(bqo_codes_bytes(fmt, 1, GROUP) + 4) / (double)GROUP;
    if (!fmt_ok(fmt)) return -1.0;
    /* bytes for one 128-weight group: codes + 2-byte scale, in bits / 128 */
    return 8.0 * (double)(bqo_codes_bytes(fmt, 1, GROUP) + 2) / (double)GROUP;
}

/* ------------------------------------------------------------------------ */
/* Decoding one weight.
 * Binary [P1; P4 §4.1]: bit k&7 of byte k>>3 (least significant bit first);
 *   bit 1 -> +1, bit 0 -> -1.
 * 2-bit slots [P2 limitations; P3 §2.4]: code c at bits 2(k&3)..2(k&3)+1 of
 *   byte k>>2; trit t = c - 1.  Reading: offset code, so c = 3 (the wasted
 *   pattern the page mentions) is invalid.
 * 5 per byte [P3 §2.4]: in group g, byte j < 25 holds trits 5j..5j+4 as
 *   v = sum_i (t_i + 1) 3^i (i = 0 least significant); byte 25 holds trits
 *   125..127 the same way.  v >= 243 (>= 27 in byte 25) is invalid.           */
int bqo_weight_code(int fmt, const uint8_t* row, int64_t k) {
    if (fmt == BQO_Q1G128) {
        int bit = (row[k >> 3] >> (k & 7)) & 1;
        return bit ? 1 : -1;
    }
    if (fmt == BQO_T2G128) {
        int c = (row[k >> 2] >> (2 * (k & 3))) & 3;
        return c == 3 ? -2 : c - 1;
    }
    if (fmt == BQO_T5P8G128) {
        int64_t g = k / GROUP;
        int kk = (int)(k % GROUP);
        int j = kk / 5, i = kk % 5;
        int v = row[g * 26 + j];
        int limit = (j < 25) ? 243 : 27;
        if (v >= limit) return -2;
        int p3 = 1;
        for (int d = 0; d < i; ++d) p3 *= 3;
        return (v / p3) % 3 - 1;
    }
    return -2;
}

static void put_code(int fmt, uint8_t* row, int64_t k, int t) {
    if (fmt == BQO_Q1G128) {
        if (t > 0) row[k >> 3] |= (uint8_t)(1u << (k & 7));
    } else if (fmt == BQO_T2G128) {
        row[k >> 2] |= (uint8_t)((t + 1) << (2 * (k & 3)));
    } else {
        int64_t g = k / GROUP;
        int kk = (int)(k % GROUP);
        int j = kk / 5, i = kk % 5;
        int p3 = 1;
        for (int d = 0; d < i; ++d) p3 *= 3;
        row[g * 26 + j] = (uint8_t)(row[g * 26 + j] + (t + 1) * p3);
    }
}

/* ------------------------------------------------------------------------ */
/* Packing.  The pages do not give the rule that maps float weights to bits
 * (weights are trained; P4 §3).  Readings taken:
 *   scale s = FP16_RNE( (sum_{i<128} |w_i|, summed in order in FP64) / 128 ),
 *     the L2-optimal scale for fixed signs (mean absolute value); a mean that
 *     rounds to infinity is an error (BQO_ERR_SCALE_RANGE);
 *   binary: bit = 1 iff w >= 0 (so +0 and -0 give +1);
 *   ternary: t = 0 if |w| <= s/2 (exact FP64 compare), else sign(w); this is
 *     clamp(round_half_even(w/s), -1, 1).
 * Given scales (scales_in) must be finite with the sign bit clear.           */
int bqo_pack(int fmt, const float* w, int64_t n, int64_t k,
             const uint16_t* scales_in, uint8_t* codes, uint16_t* scales) {
    if (!fmt_ok(fmt)) return BQO_ERR_FORMAT;
    if (n < 0 || k < 0 || k % GROUP) return BQO_ERR_SHAPE;
    if (n == 0 || k == 0) return BQO_OK;
    if (!w || !codes || !scales) return BQO_ERR_NULL;
    const int64_t G = k / GROUP;
    const int64_t row_bytes = bqo_codes_bytes(fmt, 1, k);
    memset(codes, 0, (size_t)(row_bytes * n));
    for (int64_t r = 0; r < n; ++r) {
        uint8_t* row = codes + r * row_bytes;
        for (int64_t g = 0; g < G; ++g) {
            const float* wg = w + r * k + g * GROUP;
            for (int i = 0; i < GROUP; ++i)
                if (!isfinite(wg[i])) return BQO_ERR_NONFINITE;
            uint16_t sh;
            if (scales_in) {
                sh = scales_in[r * G + g];
                if ((sh & 0x8000) || (sh & 0x7C00) == 0x7C00) return BQO_ERR_SCALE_RANGE;
            } else {
                double sum = 0.0;
                for (int i = 0; i < GROUP; ++i) sum += fabs((double)wg[i]);
                sh = bqo_double_to_half(sum / (double)GROUP);
                if ((sh & 0x7C00) == 0x7C00) return BQO_ERR_SCALE_RANGE;
            }
            scales[r * G + g] = sh;
            double s = bqo_half_to_double(sh);
            for (int i = 0; i < GROUP; ++i) {
                double wi = (double)wg[i];
                int t;
                if (fmt == BQO_Q1G128)
                    t = (wi >= 0.0) ? 1 : -1;
                else
                    t = (fabs(wi) <= s / 2.0) ? 0 : (wi > 0.0 ? 1 : -1);
                put_code(fmt, row, g * GROUP + i, t);
            }
        }
    }
    return BQO_OK;
}

int bqo_unpack(int fmt, const uint8_t* codes, int64_t n, int64_t k, int8_t* q) {
    if (!fmt_ok(fmt)) return BQO_ERR_FORMAT;
    if (n < 0 || k < 0 || k % GROUP) return BQO_ERR_SHAPE;
    if (n == 0 || k == 0) return BQO_OK;
    if (!codes || !q) return BQO_ERR_NULL;
    const int64_t row_bytes = bqo_codes_bytes(fmt, 1, k);
    for (int64_t r = 0; r < n; ++r)
        for (int64_t kk = 0; kk < k; ++kk) {
            int t = bqo_weight_code(fmt, codes + r * row_bytes, kk);
            if (t == -2) return BQO_ERR_FORMAT;
            q[r * k + kk] = (int8_t)t;
        }
    return BQO_OK;
}

/* ------------------------------------------------------------------------ */
/* Product [P4 §4.1: effective weight = signed code x group FP16 scale, times
 * the activation]: y = sum_g s_g * sum_{k in g} q_k x_k, all in FP64.
 * bound = sum_k |s_g(k) x_k| is the scale of the stated tolerance.            */
static int one_row(int fmt, const uint8_t* row, const uint16_t* srow, int64_t k,
                   const uint16_t* xb, double* y, double* bound) {
    const int64_t G = k / GROUP;
    double acc = 0.0, bnd = 0.0;
    for (int64_t g = 0; g < G; ++g) {
        double s = bqo_half_to_double(srow[g]);
        double p = 0.0, ax = 0.0;
        for (int i = 0; i < GROUP; ++i) {
            int64_t kk = g * GROUP + i;
            int t = bqo_weight_code(fmt, row, kk);
            if (t == -2) return BQO_ERR_FORMAT;
            double x = bqo_bf16_to_double(xb[kk]);
            p += (double)t * x;
            ax += fabs(x);
        }
        acc += s * p;
        bnd += fabs(s) * ax;
    }
    *y = acc;
    *bound = bnd;
    return BQO_OK;
}

int bqo_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

int bqo_matmul_rows(int fmt, const uint8_t* codes, const uint16_t* scales,
                    int64_t n, int64_t k, const uint16_t* x, int64_t batch,
                    const int64_t* rows, int64_t nrows,
                    double* y, double* bound, int nthreads) {
    if (!fmt_ok(fmt)) return BQO_ERR_FORMAT;
    if (n < 0 || k < 0 || k % GROUP || batch < 0 || nrows < 0) return BQO_ERR_SHAPE;
    if (nrows == 0 || batch == 0) return BQO_OK;
    if (!codes || !scales || !x || !rows || !y || !bound) return BQO_ERR_NULL;
    for (int64_t i = 0; i < nrows; ++i)
        if (rows[i] < 0 || rows[i] >= n) return BQO_ERR_SHAPE;
    const int64_t row_bytes = bqo_codes_bytes(fmt, 1, k);
    const int64_t G = k / GROUP;
    int status = BQO_OK;
#ifdef _OPENMP
    int nt = nthreads > 0 ? nthreads : omp_get_max_threads();
#pragma omp parallel for num_threads(nt) schedule(dynamic, 16)
#endif
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t r = rows[i];
        for (int64_t b = 0; b < batch; ++b) {
            int st = one_row(fmt, codes + r * row_bytes, scales + r * G, k,
                             x + b * k, &y[b * nrows + i], &bound[b * nrows + i]);
            if (st != BQO_OK) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
                status = st;
            }
        }
    }
    (void)nthreads;
    return status;
}

int bqo_matmul(int fmt, const uint8_t* codes, const uint16_t* scales,
               int64_t n, int64_t k, const uint16_t* x, int64_t batch,
               double* y, double* bound, int nthreads) {
    if (!fmt_ok(fmt)) return BQO_ERR_FORMAT;
    if (n < 0 || k < 0 || k % GROUP || batch < 0) return BQO_ERR_SHAPE;
    if (n == 0 || batch == 0) return BQO_OK;
    if (!codes || !scales || !x || !y || !bound) return BQO_ERR_NULL;
    const int64_t row_bytes = bqo_codes_bytes(fmt, 1, k);
    const int64_t G = k / GROUP;
    int status = BQO_OK;
#ifdef _OPENMP
    int nt = nthreads > 0 ? nthreads : omp_get_max_threads();
#pragma omp parallel for num_threads(nt) schedule(dynamic, 16)
#endif
    for (int64_t r = 0; r < n; ++r) {
        for (int64_t b = 0; b < batch; ++b) {
            int st = one_row(fmt, codes + r * row_bytes, scales + r * G, k,
                             x + b * k, &y[b * n + r], &bound[b * n + r]);
            if (st != BQO_OK) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
                status = st;
            }
        }
    }
    (void)nthreads;
    return status;
}

/* ------------------------------------------------------------ SwiGLU */
/* silu(v) = v * sigma(v), sigma(v) = 1 / (1 + e^-v); the gate value times the
 * matching up value, rounded once to BF16. */
int bqo_swiglu(const double* h, int64_t batch, int64_t inter, uint16_t* act_bf16, double* act_f64) {
    if (batch < 0 || inter < 0) return BQO_ERR_SHAPE;
    if (batch == 0 || inter == 0) return BQO_OK;
    if (!h || !act_bf16) return BQO_ERR_NULL;
    for (int64_t b = 0; b < batch; ++b) {
        const double* hb = h + b * 2 * inter;
        for (int64_t j = 0; j < inter; ++j) {
            const double g = hb[j], u = hb[inter + j];
            const double a = (g / (1.0 + exp(-g))) * u;
            act_bf16[b * inter + j] = bqo_double_to_bf16(a);
            if (act_f64) act_f64[b * inter + j] = a;
        }
    }
    return BQO_OK;
}

/* ------------------------------------------------------------ embedding rows */
/* Embedding lookup on a low-bit table ("1-bit Bonsai 8B" notes, section 3 and
 * Table 1: the embedding layer is low-bit too): row ids[i] of the table,
 * dequantised as s * q in FP64 (exact) and rounded once to BF16. */
int bqo_embed_rows(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                   const int32_t* ids, int64_t count, uint16_t* out_bf16) {
    if (fmt != BQO_Q1G128 && fmt != BQO_T2G128 && fmt != BQO_T5P8G128) return BQO_ERR_FORMAT;
    if (n < 0 || k < 0 || k % GROUP || count < 0) return BQO_ERR_SHAPE;
    if (count == 0 || k == 0) return BQO_OK;
    if (!codes || !scales || !ids || !out_bf16) return BQO_ERR_NULL;
    const int64_t row_bytes = bqo_codes_bytes(fmt, 1, k);
    const int64_t G = k / GROUP;
    for (int64_t i = 0; i < count; ++i) {
        const int64_t r = ids[i];
        if (r < 0 || r >= n) return BQO_ERR_SHAPE;
        const uint8_t* row = codes + r * row_bytes;
        for (int64_t kk = 0; kk < k; ++kk) {
            const double s = bqo_half_to_double(scales[r * G + kk / GROUP]);
            const int q = bqo_weight_code(fmt, row, kk);
            out_bf16[i * k + kk] = bqo_double_to_bf16(s * (double)q);
        }
    }
    return BQO_OK;
}

/* ------------------------------------------------------------ affine 1-bit */
static int affine_bit(const uint8_t* row, int64_t k) { return (row[k >> 3] >> (k & 7)) & 1; }

int bqo_pack_affine(const float* w, int64_t n, int64_t k, const uint16_t* params_in,
                    uint8_t* codes, uint16_t* params) {
    if (n < 0 || k < 0 || k % GROUP) return BQO_ERR_SHAPE;
    if (n == 0 || k == 0) return BQO_OK;
    if (!w || !codes || !params) return BQO_ERR_NULL;
    const int64_t G = k / GROUP;
    memset(codes, 0, (size_t)(n * (k / 8)));
    for (int64_t r = 0; r < n; ++r) {
        for (int64_t g = 0; g < G; ++g) {
            const float* wg = w + r * k + g * GROUP;
            for (int i = 0; i < GROUP; ++i)
                if (!isfinite(wg[i])) return BQO_ERR_NONFINITE;
            uint16_t sh, zh;
            if (params_in) {
                sh = params_in[(r * G + g) * 2];
                zh = params_in[(r * G + g) * 2 + 1];
                if ((sh & 0x8000) || (sh & 0x7C00) == 0x7C00 || (zh & 0x7C00) == 0x7C00) return BQO_ERR_SCALE_RANGE;
            } else {
                double lo = wg[0], hi = wg[0];
                for (int i = 1; i < GROUP; ++i) {
                    if (wg[i] < lo) lo = wg[i];
                    if (wg[i] > hi) hi = wg[i];
                }
                zh = bqo_double_to_half(lo);
                sh = bqo_double_to_half(hi - lo); /* exact in FP64 for two floats */
                if ((sh & 0x7C00) == 0x7C00 || (zh & 0x7C00) == 0x7C00) return BQO_ERR_SCALE_RANGE;
            }
            params[(r * G + g) * 2] = sh;
            params[(r * G + g) * 2 + 1] = zh;
            const double sv = bqo_half_to_double(sh), zv = bqo_half_to_double(zh);
            uint8_t* row = codes + r * (k / 8);
            for (int i = 0; i < GROUP; ++i) {
                const int64_t kk = g * GROUP + i;
                if ((double)wg[i] - zv > sv / 2.0) row[kk >> 3] |= (uint8_t)(1u << (kk & 7));
            }
        }
    }
    return BQO_OK;
}

int bqo_matmul_affine(const uint8_t* codes, const uint16_t* params, int64_t n, int64_t k,
                      const uint16_t* x, int64_t batch, const int64_t* rows, int64_t nrows,
                      double* y, double* bound, int nthreads) {
    if (n < 0 || k < 0 || k % GROUP || batch < 0) return BQO_ERR_SHAPE;
    const int64_t R = rows ? nrows : n;
    if (R < 0) return BQO_ERR_SHAPE;
    if (R == 0 || batch == 0) return BQO_OK;
    if (!codes || !params || !x || !y || !bound) return BQO_ERR_NULL;
    if (rows)
        for (int64_t i = 0; i < R; ++i)
            if (rows[i] < 0 || rows[i] >= n) return BQO_ERR_SHAPE;
    const int64_t G = k / GROUP;
#ifdef _OPENMP
    int nt = nthreads > 0 ? nthreads : omp_get_max_threads();
#pragma omp parallel for num_threads(nt) schedule(dynamic, 16)
#endif
    for (int64_t i = 0; i < R; ++i) {
        const int64_t r = rows ? rows[i] : i;
        const uint8_t* row = codes + r * (k / 8);
        for (int64_t b = 0; b < batch; ++b) {
            const uint16_t* xb = x + b * k;
            double acc = 0.0, bnd = 0.0;
            for (int64_t g = 0; g < G; ++g) {
                const double sv = bqo_half_to_double(params[(r * G + g) * 2]);
                const double zv = bqo_half_to_double(params[(r * G + g) * 2 + 1]);
                double ax = 0.0;
                for (int j = 0; j < GROUP; ++j) {
                    const int64_t kk = g * GROUP + j;
                    const double xv = bqo_bf16_to_double(xb[kk]);
                    acc += (sv * (double)affine_bit(row, kk) + zv) * xv;
                    ax += fabs(xv);
                }
                bnd += (fabs(sv) + fabs(zv)) * ax;
            }
            y[b * R + i] = acc;
            bound[b * R + i] = bnd;
        }
    }
    (void)nthreads;
    return BQO_OK;
}

int bqo_embed_rows_affine(const uint8_t* codes, const uint16_t* params, int64_t n, int64_t k,
                          const int32_t* ids, int64_t count, uint16_t* out_bf16) {
    if (n < 0 || k < 0 || k % GROUP || count < 0) return BQO_ERR_SHAPE;
    if (count == 0 || k == 0) return BQO_OK;
    if (!codes || !params || !ids || !out_bf16) return BQO_ERR_NULL;
    const int64_t G = k / GROUP;
    for (int64_t i = 0; i < count; ++i) {
        const int64_t r = ids[i];
        if (r < 0 || r >= n) return BQO_ERR_SHAPE;
        for (int64_t kk = 0; kk < k; ++kk) {
            const int64_t g = kk / GROUP;
            const double sv = bqo_half_to_double(params[(r * G + g) * 2]);
            const double zv = bqo_half_to_double(params[(r * G + g) * 2 + 1]);
            out_bf16[i * k + kk] = bqo_double_to_bf16(sv * (double)affine_bit(codes + r * (k / 8), kk) + zv);
        }
    }
    return BQO_OK;
}
