/*
 * bq_oracle.h -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, obviously-correct CPU definitions (FP64) of what the binary /
 * ternary g128 weight path computes.  Only tests/, __graft_entry__.smoke() and
 * bench.py's cpu_baseline / reference arm may load this library.  It shares no
 * code, header, table or constant with the CUDA library under
 * ternary_g128_weight_b200/; the enum values below are restated here on
 * purpose and are checked against the product's values by the tests.
 *
 * Sources (web pages on "Bonsai" 1-bit / ternary g128 models):
 *   [P1] "Bonsai-27B-mlx-1bit ... Binary g128 权重表示" -- section on the Binary
 *        g128 weight representation: one sign bit per weight (0 -> -scale,
 *        1 -> +scale), one FP16 scale shared by 128 weights, 1.125 bits/weight.
 *   [P2] "Ternary Bonsai" -- section "什么是Ternary Bonsai技术": trits
 *        {-1,0,+1} times an FP16 scale per 128 weights, ~1.71 bits/weight;
 *        limitations: stored in 2-bit slots today.
 *   [P3] "把 27B 模型压到 4GB 跑在手机上" -- section 2.4: the 2-bit slot code
 *        wastes one pattern; 5 trits fit in 8 bits (3^5 = 243 <= 256).
 *   [P4] "1-bit Bonsai 8B" whitepaper notes -- section 4.1 (Q1_0_g128: bits in
 *        {0,1} mapped to signed values times the group FP16 scale, decoded
 *        inline in the matmul) and Table 2 (package sizes).
 */
#ifndef BQ_ORACLE_H
#define BQ_ORACLE_H
#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { BQO_OK = 0, BQO_ERR_NULL = 1, BQO_ERR_SHAPE = 2, BQO_ERR_ALIGN = 3,
       BQO_ERR_NONFINITE = 4, BQO_ERR_SCALE_RANGE = 5, BQO_ERR_FORMAT = 6 };
enum { BQO_Q1G128 = 1, BQO_T2G128 = 2, BQO_T5P8G128 = 3, BQO_A1G128 = 4 };

/* IEEE-754 binary16 and bfloat16, written from the encoding definitions. */
double   bqo_half_to_double(uint16_t h);
uint16_t bqo_double_to_half(double v);      /* round to nearest, ties to even */
double   bqo_bf16_to_double(uint16_t b);
uint16_t bqo_double_to_bf16(double v);      /* round to nearest, ties to even */

/* Storage sizes and bits per weight (codes + one FP16 scale per 128). */
int64_t bqo_codes_bytes(int fmt, int64_t n, int64_t k);
int64_t bqo_scales_bytes(int64_t n, int64_t k);
double  bqo_effective_bits(int fmt);

/* Trit / sign code of weight k of one packed row: -1, 0 or +1; -2 if the
 * stored code is not a valid code of the format. */
int bqo_weight_code(int fmt, const uint8_t* row_codes, int64_t k);

/* float W[n][k] -> codes + FP16 scales.  scales_in (may be NULL) gives the
 * scales instead of the mean-|w| rule. */
int bqo_pack(int fmt, const float* w, int64_t n, int64_t k,
             const uint16_t* scales_in, uint8_t* codes, uint16_t* scales);

/* codes -> q[n][k] in {-1,0,+1}. */
int bqo_unpack(int fmt, const uint8_t* codes, int64_t n, int64_t k, int8_t* q);

/* y[b][r] = sum_g s[r][g] * sum_{k in g} q[r][k] * x[b][k]  (FP64)
 * bound[b][r] = sum_k |s[r][g(k)] * x[b][k]|                 (FP64)
 * for every row r (bqo_matmul) or for the rows listed (bqo_matmul_rows, output
 * [batch][nrows]).  x is BF16 [batch][k].  nthreads <= 0 uses all cores. */
int bqo_matmul(int fmt, const uint8_t* codes, const uint16_t* scales,
               int64_t n, int64_t k, const uint16_t* x, int64_t batch,
               double* y, double* bound, int nthreads);
int bqo_matmul_rows(int fmt, const uint8_t* codes, const uint16_t* scales,
                    int64_t n, int64_t k, const uint16_t* x, int64_t batch,
                    const int64_t* rows, int64_t nrows,
                    double* y, double* bound, int nthreads);

/* SwiGLU activation of a gated MLP block (the 8B whitepaper notes, Table 1:
 * SwiGLU feed-forward): for h[b] = [gate | up] of length 2 * inter (the FP64
 * product of the concatenated gate and up matrices),
 *   act[b][j] = BF16_RNE( silu(h[b][j]) * h[b][inter + j] ),
 *   silu(v) = v / (1 + exp(-v)),
 * computed in FP64; act_f64 (may be NULL) receives the unrounded values. */
int bqo_swiglu(const double* h, int64_t batch, int64_t inter, uint16_t* act_bf16, double* act_f64);

/* Embedding lookup: out[i][k] = BF16_RNE(s[ids[i]][k/128] * q[ids[i]][k])
 * (the product in FP64 is exact), for i < count.  An id outside [0, n) is
 * BQO_ERR_SHAPE. */
int bqo_embed_rows(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                   const int32_t* ids, int64_t count, uint16_t* out_bf16);

/* Affine 1-bit g128, the MLX-style variant ("Bonsai-27B-mlx-1bit ... Binary
 * g128", section "MLX打包优化": MLX's grouped low-bit format stores a scale and a
 * bias per group; "1-bit Bonsai 8B" notes, Table 2: the MLX 1-bit (g128)
 * package): w' = s * b + z, b in {0, 1} stored as the binary format stores its
 * bits, one FP16 pair (s, z) per 128 weights in params [N][G][2].
 * Packing (a reading; the pages give no rule): z = FP16_RNE(min w),
 * s = FP16_RNE(max w - min w), b = 1 iff w - z > s/2 (FP64, a tie gives 0),
 * i.e. round_half_even((w - z) / s) in {0, 1}.  params_in (or NULL): given
 * pairs, s finite without its sign bit, z finite.
 * Product: y = sum_g sum_{k in g} (s_g b_k + z_g) x_k (FP64) for the rows listed
 * (rows == NULL: every row, output [batch][n]); bound = sum_g (|s_g| + |z_g|)
 * sum_{k in g} |x_k|, the scale of the tolerance (over every k, as for the
 * ternary formats).
 * Embedding: out[i][k] = BF16_RNE(s b + z) of row ids[i] (FP64 exact before the
 * rounding). */
int bqo_pack_affine(const float* w, int64_t n, int64_t k, const uint16_t* params_in,
                    uint8_t* codes, uint16_t* params);
int bqo_matmul_affine(const uint8_t* codes, const uint16_t* params, int64_t n, int64_t k,
                      const uint16_t* x, int64_t batch, const int64_t* rows, int64_t nrows,
                      double* y, double* bound, int nthreads);
int bqo_embed_rows_affine(const uint8_t* codes, const uint16_t* params, int64_t n, int64_t k,
                          const int32_t* ids, int64_t count, uint16_t* out_bf16);

/* Number of OpenMP threads a call with nthreads <= 0 would use. */
int bqo_max_threads(void);

#ifdef __cplusplus
}
#endif
#endif
