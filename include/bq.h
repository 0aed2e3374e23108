/*
 * bq.h -- C ABI of the binary / ternary g128 weight library for NVIDIA B200
 * (sm_100a).
 *
 * What it computes.  End-to-end low-bit weights as described on the pages
 *   "Bonsai-27B-mlx-1bit ... Binary g128 权重表示" (section "Binary g128权重表示原理"),
 *   "Ternary Bonsai" (section "什么是Ternary Bonsai技术"),
 *   "把 27B 模型压到 4GB 跑在手机上" (section 2.4, trit storage), and
 *   "1-bit Bonsai 8B" notes (section 2 "内存带宽是真正的瓶颈", section 4.1 Q1_0_g128,
 *   Table 3 tg128 / pp512):
 * every weight is a code q in {-1,+1} (binary) or {-1,0,+1} (ternary), every
 * 128 consecutive weights of a row share one FP16 scale s, and the effective
 * weight is s*q.  Products decode the codes inside the kernel; no FP16 copy of
 * W is ever written to memory.
 *
 * Shapes and layouts (all row-major, no padding between rows):
 *   W        N x K, K % 128 == 0, G = K/128 groups per row.
 *   scales   uint16 FP16 bit patterns [N][G]; scales[r][g] covers weights
 *            r, 128g .. 128g+127.
 *   codes    BQ_Q1G128  : [N][K/8]  bytes; weight k at bit (k&7) of byte k>>3,
 *                         bit 1 -> +1, bit 0 -> -1.          1.125 bits/weight
 *            BQ_T2G128  : [N][K/4]  bytes; code c = q+1 in bits 2(k&3)..+1 of
 *                         byte k>>2; c == 3 is not a valid code. 2.125 bits/weight
 *            BQ_T5P8G128: [N][26*G] bytes; in group g, byte j < 25 holds
 *                         v = sum_{i<5} (q_{128g+5j+i}+1) 3^i, byte 25 holds the
 *                         last three codes the same way.      1.75 bits/weight
 *            BQ_A1G128  : the BQ_Q1G128 bit layout, but bit b means s*b + z: the
 *                         affine variant MLX packs ("Bonsai-27B-mlx-1bit ... Binary
 *                         g128", section "MLX打包优化": a scale and a bias per
 *                         group).  Its `scales` array holds FP16 (s, z) pairs
 *                         [N][G][2].                          1.25 bits/weight
 *                         Supported by the packer, bq_gemv / bq_gemv_noalloc on
 *                         the row-owning path (batch <= 8, K % 1024 == 0) and
 *                         bq_embed_rows; bq_gemm and bq_gemv_chain return
 *                         BQ_ERR_FORMAT.  Tolerance scale for this format:
 *                         sum_k (|s| + |z|) |x_k| over every k.
 *   x        BF16 bit patterns [B][K] (GEMV) or [T][K] (GEMM), contiguous.
 *   y        [B][N] (GEMV, BF16 or F32) or [T][N] (GEMM, BF16).
 *
 * Ownership.  Every pointer argument of the compute calls is a DEVICE pointer
 * owned by the caller.  The library allocates no memory and keeps no pointer
 * after a call returns.  Workspaces are caller-allocated device buffers of at
 * least the size the matching *_workspace_bytes call reports.
 *
 * Streams.  `stream` is a cudaStream_t passed as void* (NULL = the legacy
 * default stream).  bq_gemv and bq_gemm only enqueue work and return; they do
 * not synchronise.  The packers synchronise `stream` before returning because
 * their status (non-finite input, scale overflow) is produced on the device.
 *
 * Errors.  Argument errors are detected on the host before anything is
 * launched and returned synchronously; nothing is written.  A launch failure
 * returns BQ_ERR_CUDA.  Asynchronous faults and device-side time-outs of
 * bounded waits surface through bq_check().  Invalid codes (a 2-bit code of 3,
 * a base-3 byte >= 243) give unspecified output values, never a fault.
 *
 * Precision.  Activations are read as BF16, products accumulate in FP32 with
 * one scale multiply per group; every output satisfies
 *   |y - y_exact| <= 2e-3 * sum_k |s_{g(k)} x_k|
 * plus the final rounding to the output type (for BF16 output at most
 * 2^-8 |y|).
 */
#ifndef BQ_H
#define BQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BQ_OK = 0,
    BQ_ERR_NULL = 1,        /* a required pointer is NULL */
    BQ_ERR_SHAPE = 2,       /* K % 128 != 0, a negative size, batch out of range */
    BQ_ERR_ALIGN = 3,       /* a pointer is not aligned as documented */
    BQ_ERR_NONFINITE = 4,   /* packer input holds NaN or +-Inf */
    BQ_ERR_SCALE_RANGE = 5, /* a scale would exceed FP16, or a given scale is negative / non-finite */
    BQ_ERR_FORMAT = 6,      /* unknown format or output dtype */
    BQ_ERR_CUDA = 7,        /* a CUDA runtime call failed (launch error, sticky fault) */
    BQ_ERR_TIMEOUT = 8,     /* a bounded device wait gave up (reported by bq_check) */
    BQ_ERR_WORKSPACE = 9    /* workspace NULL or smaller than *_workspace_bytes */
} bq_status;

typedef enum { BQ_Q1G128 = 1, BQ_T2G128 = 2, BQ_T5P8G128 = 3, BQ_A1G128 = 4 } bq_format;
typedef enum { BQ_BF16 = 0, BQ_F32 = 1 } bq_dtype;

#define BQ_GROUP 128
#define BQ_MAX_BATCH 16

/* ------------------------------------------------------------------ sizes */
/* Bytes of the code array for an N x K matrix; -1 for an invalid format or
 * shape (negative size or K % 128 != 0).  Binary: one bit per weight, packed
 * ("1-bit Bonsai 8B" notes, section 4.1: the {0,1} bits are stored packed,
 * 1 bit per weight).  2-bit slots: one 2-bit code per trit; 5 trits per byte:
 * 3^5 = 243 <= 256 ("把 27B 模型压到 4GB" section 2.4 on both ternary
 * storages). */
int64_t bq_codes_bytes(int fmt, int64_t n, int64_t k);
/* Bytes of the group parameters of a format: N * (K/128) * 2 (one FP16 scale per
 * group), or N * (K/128) * 4 for BQ_A1G128 ((scale, bias) pairs); -1 if invalid. */
int64_t bq_group_params_bytes(int fmt, int64_t n, int64_t k);
/* Bytes of the FP16 scale array, N * (K/128) * 2; -1 for an invalid shape.
 * One FP16 scale per 128 consecutive weights ("Bonsai-27B-mlx-1bit ...
 * Binary g128", section "Binary g128权重表示原理"). */
int64_t bq_scales_bytes(int64_t n, int64_t k);
/* Storage bits per weight including the scale: 1.125, 2.125, 1.75; -1 if
 * invalid.  1.125 = 1 + 16/128 is the binary g128 figure of the "1-bit Bonsai
 * 8B" notes (section 4.1, Table 2); the ternary page's 1.71 bits ("Ternary
 * Bonsai", section "什么是Ternary Bonsai技术") is the entropy log2(3) + 16/128,
 * which no byte-addressed storage here reaches. */
double bq_effective_bits(int fmt);

/* ---------------------------------------------------------------- packers */
/* Float weights -> codes + FP16 scales (one thread per 128-weight group).
 * The codes: bq_pack_q1g128 writes bit 1 for +scale and bit 0 for -scale
 * ("Bonsai-27B-mlx-1bit ... Binary g128", section "Binary g128权重表示原理");
 * bq_pack_t2g128 / bq_pack_t5p8 write trits {-1, 0, +1} in 2-bit slots / five
 * per byte ("Ternary Bonsai", section "什么是Ternary Bonsai技术"; "把 27B 模型压到
 * 4GB" section 2.4).
 * Reading of the pages, which do not state the rule for trained weights:
 *   s = FP16 round-to-nearest-even of (sum of |w| over the group, summed in
 *       order in FP64) / 128, unless `scales_in` gives the scales;
 *   binary : q = +1 if w >= 0 (both zeros give +1), else -1;
 *   ternary: q = 0 if |w| <= s/2, else sign(w)  (= clamp(round-half-even(w/s))).
 * w        device float32 [N][K], 16-byte aligned.
 * scales_in device FP16 [N][G] or NULL; each must be finite and non-negative.
 * codes    device [bq_codes_bytes] bytes; scales device FP16 [N][G].
 * Returns BQ_ERR_NONFINITE / BQ_ERR_SCALE_RANGE if any group fails (then the
 * outputs are unspecified).  Synchronises `stream`.  The result is bit-exact
 * with the reference definition. */
bq_status bq_pack_q1g128(const float* w, int64_t n, int64_t k, const uint16_t* scales_in,
                         uint8_t* codes, uint16_t* scales, void* stream);
bq_status bq_pack_t2g128(const float* w, int64_t n, int64_t k, const uint16_t* scales_in,
                         uint8_t* codes, uint16_t* scales, void* stream);
bq_status bq_pack_t5p8(const float* w, int64_t n, int64_t k, const uint16_t* scales_in,
                       uint8_t* codes, uint16_t* scales, void* stream);
/* Affine 1-bit packer (BQ_A1G128).  Reading of the pages, which give no rule:
 *   z = FP16_RNE(min w), s = FP16_RNE(max w - min w) (the difference exact in
 *   FP64), b = 1 iff w - z > s/2 (FP64; a tie gives 0), unless params_in gives
 *   the (s, z) pairs ([N][G][2] FP16: s finite with its sign bit clear, z
 *   finite).  params: device FP16 [N][G][2].  Errors and synchronisation as the
 *   other packers; the result is bit-exact with the reference definition. */
bq_status bq_pack_a1g128(const float* w, int64_t n, int64_t k, const uint16_t* params_in,
                         uint8_t* codes, uint16_t* params, void* stream);

/* ------------------------------------------------------------------- GEMV */
/* Workspace bytes bq_gemv needs for this call shape (0 when none is needed);
 * -1 for an invalid format or shape. */
int64_t bq_gemv_workspace_bytes(int fmt, int64_t n, int64_t k, int batch);

/* Number of kernels one bq_gemv (or bq_gemv_noalloc) call of this shape
 * launches (0 for an empty shape); -1 for an invalid format or shape.  An
 * introspection helper for callers that count launches (graph building,
 * benchmarks); it launches nothing. */
int bq_gemv_launches(int fmt, int64_t n, int64_t k, int batch);

/* y[b][r] = sum_g s[r][g] * sum_{k in g} q[r][k] * x[b][k],   b < batch <= 16.
 * The weight-streaming decode product ("1-bit Bonsai 8B" section 2: token
 * generation is bound by streaming the weights; section 4.1: codes decoded
 * inline in the matmul).
 * codes/scales as above; x BF16 [batch][K]; y [batch][N] of y_dtype.  The
 * base of every array (codes, scales, x, y) must be 16-byte aligned.
 * workspace: device buffer of >= bq_gemv_workspace_bytes bytes (may be NULL
 * when that is 0), 256-byte aligned; its contents on entry do not matter.
 * Asynchronous on `stream`.
 * Kernel choice (the same for bq_gemv_noalloc and for bq_gemm with T <= 4):
 * K % 1024 == 0 with binary or 2-bit ternary codes at batch 5..16, or 5-trit
 * codes at batch 9..16, runs the wide-batch GEMV (FP16 effective weights
 * +-s / {-s,0,+s} built in registers, x pre-scaled per row to FP16, one
 * launch, no workspace) when its FP16 activations (2 K bytes per row, rows
 * padded to 8 or 16) and a ring of two weight slots fit in shared memory;
 * batch <= 8 and K % 1024 == 0 otherwise run the row-owning
 * tensor-core GEMV (all three formats, one launch, no workspace) when its
 * activation operand and a ring of at least two weight slots fit in shared
 * memory; otherwise binary and 2-bit ternary at batch <= 4 run the split-K
 * tensor-core GEMV (workspace), and the rest (K % 1024 != 0, operands too
 * large) the tcgen05 GEMM with T = batch
 * (workspace for the FP16 activations).  A shape
 * no kernel takes (K > 2^28, or N >= 2^31) returns BQ_ERR_SHAPE.
 * bq_gemv_workspace_bytes and bq_gemv_launches report the chosen path (-1 for
 * such a shape). */
bq_status bq_gemv(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                  const uint16_t* x, int batch, void* y, int y_dtype,
                  void* workspace, size_t workspace_bytes, void* stream);

/* Allocation-free GEMV.  (The pages have no counterpart: this serves callers,
 * not the method.)  Same product, arguments and layouts as bq_gemv, but with no
 * workspace argument: for callers that cannot allocate device memory where they
 * run it -- a host that owns all device memory and passes a plugin only its
 * inputs and outputs, or a path where cudaMalloc's possible device
 * synchronisation is not acceptable.  The scratch it needs lives in one fixed
 * array of BQ_NOALLOC_SCRATCH_BYTES bytes inside the library, held on every GPU
 * that loads the library until the process exits.  Shapes whose scratch need
 * (bq_gemv_workspace_bytes) exceeds that size return BQ_ERR_WORKSPACE and
 * nothing is launched.  The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress, with that device current); make that first
 * call before capturing a stream.  All calls share the array and it keeps the
 * last call's contents (what must start at zero is cleared by every call); two
 * calls that overlap on the GPU race on it, so order them on one stream.
 * Allocates nothing (no cudaMalloc / cudaFree).  Asynchronous on `stream`. */
#define BQ_NOALLOC_SCRATCH_BYTES (4u << 20)
bq_status bq_gemv_noalloc(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                          const uint16_t* x, int batch, void* y, int y_dtype, void* stream);

/* -------------------------------------------------------------- embedding */
/* Embedding lookup on a low-bit table ("1-bit Bonsai 8B" notes, section 3 and
 * Table 1: the embedding layer is low-bit too):
 *   out[i][k] = BF16_RNE(s[ids[i]][k/128] * q[ids[i]][k]),   i < count,
 * exact up to the one rounding of the FP16 scale to BF16.  codes/scales: the
 * N x K table as above (16-byte aligned); ids: device int32 [count] (4-byte
 * aligned); out: device BF16 [count][K] (16-byte aligned).  An id outside
 * [0, N) gives a zero row and makes bq_check() report BQ_ERR_SHAPE (the ids
 * live on the device, so the host cannot check them).  Asynchronous on
 * `stream`. */
bq_status bq_embed_rows(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                        const int32_t* ids, int64_t count, uint16_t* out, void* stream);

/* --------------------------------------------------------- layer chains */
/* One product of a chain (see bq_gemv_chain).  All pointers are device
 * pointers; codes/scales/x 16-byte aligned as for bq_gemv. */
typedef struct {
    const uint8_t* codes;   /* W, N x K, the chain's format */
    const uint16_t* scales; /* FP16 [N][K/128] */
    int64_t n, k;           /* K % 1024 == 0 */
    const uint16_t* x;      /* BF16 [batch][K]; may be an earlier step's y */
    void* y;                /* swiglu == 0: [batch][N] of y_dtype; swiglu == 1: BF16 [batch][N/2] */
    int y_dtype;            /* BQ_BF16 or BQ_F32 (swiglu == 0); a y that a later step
                               reads as its x must be BQ_BF16 */
    int swiglu;             /* 0: y = W x.  1: W = [gate; up] (N = 2 I, I % 16 == 0):
                               y[b][j] = BF16_RNE(silu(g_j) * u_j), g = W_gate x,
                               u = W_up x, silu(v) = v / (1 + e^-v) */
} bq_chain_step;

#define BQ_MAX_CHAIN_STEPS 8

/* Workspace bytes of bq_gemv_chain: its grid-barrier counters (256). */
int64_t bq_gemv_chain_workspace_bytes(void);

/* The products of one decoder layer, in order, in ONE persistent launch ("1-bit
 * Bonsai 8B" notes, Table 1: the attention projections and the SwiGLU
 * feed-forward of each block; section 2: decode is bound by streaming the
 * weights).  steps[0..nsteps) (HOST array, read during the call) run one
 * after another with a device-wide barrier between them: every step sees all
 * outputs of the steps before it, so a step's x may be an earlier step's y (for
 * example the gated MLP: gate|up with swiglu = 1 writing act, then down with
 * x = act).  Each product is the bq_gemv product (same tolerance); a SwiGLU
 * step rounds its output once, to BF16.  One CTA per SM streams every step's
 * weights back to back, so the weights of the next step arrive while the
 * current one computes.
 * fmt for all steps; 1 <= nsteps <= BQ_MAX_CHAIN_STEPS; batch 1..8 (limited by
 * shared memory: the activation operand of the largest K must fit, else
 * BQ_ERR_SHAPE).
 * workspace: >= bq_gemv_chain_workspace_bytes() device bytes, 16-byte aligned,
 * ZERO-FILLED before its first use; every call leaves it zero.  Calls that
 * share a workspace must not overlap on the GPU.  After bq_check() reports
 * BQ_ERR_TIMEOUT, zero it again.
 * The launch is cooperative: it fails (BQ_ERR_CUDA) where one CTA per SM
 * cannot be resident.  Asynchronous on `stream`. */
bq_status bq_gemv_chain(int fmt, const bq_chain_step* steps, int nsteps, int batch,
                        void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------- GEMM */
/* Workspace bytes bq_gemm needs for T tokens (0 if none); -1 if invalid. */
int64_t bq_gemm_workspace_bytes(int fmt, int64_t n, int64_t k, int64_t t);

/* Number of kernels one bq_gemm call of this shape launches (0 for an empty
 * shape); -1 if invalid.  Introspection only; launches nothing. */
int bq_gemm_launches(int fmt, int64_t n, int64_t k, int64_t t);

/* Prefill: Y[t][r] = sum_k X[t][k] * s[r][g(k)] q[r][k] for t < T, BF16 out
 * ("1-bit Bonsai 8B" summary section 3 and Table 3 pp512: prompt processing is
 * a dense contraction).  For T <= 16 this is bq_gemv with batch = T.  Larger T
 * runs a tensor-core (tcgen05) kernel that dequantises W tiles on chip to FP16
 * s*q (exact) and multiplies by X converted to FP16 with a per-token
 * power-of-two pre-scale (exact for every BF16 value within 2^-31 of the
 * token's largest magnitude), accumulating in FP32.
 * X BF16 [T][K] 16-byte aligned; Y BF16 [T][N] 16-byte aligned; workspace as
 * bq_gemm_workspace_bytes, 256-byte aligned (FP16 activations and, where K is
 * split over CTAs, FP32 partial tiles, rewritten by every call: calls that
 * share a workspace must not overlap on the GPU).  Asynchronous on `stream`. */
bq_status bq_gemm(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                  const uint16_t* x, int64_t t, uint16_t* y,
                  void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------- 4-bit KV cache */
/* A 4-bit KV cache for decode attention ("Bonsai-27B-mlx-1bit ... Binary
 * g128", sections "峰值内存管理" and "KV压缩潜力": the KV cache is quantised to
 * 4 bits for long contexts; "Ternary Bonsai", hybrid-attention section: 4-bit
 * KV-cache quantisation; "1-bit Bonsai 8B" notes, Table 1: grouped-query
 * attention, 32 query / 8 KV heads).  The pages fix the bit width only; the
 * format is this library's reading:
 *   every cached K or V vector of head dimension D (128 or 256) is cut into
 *   groups of 128 values, each stored as 64 bytes of 4-bit codes (value 2i in
 *   the low nibble of byte i) and one 32-bit word (FP16 scale s in bits 0..15,
 *   FP16 bias z in bits 16..31), min-max affine with 16 levels:
 *     s = FP16_RNE((max - min) / 15), z = FP16_RNE(min)  (the quotient in FP64),
 *     c = clamp(rint((x - z) / s), 0, 15)  (in FP64; c = 0 when s == 0),
 *     value = s c + z.                                  4.25 bits per value
 * A group holding NaN / Inf is stored as zeros (s = z = 0, codes 0) and
 * bq_check() reports BQ_ERR_NONFINITE; one whose s or z overflows FP16 the
 * same, with BQ_ERR_SCALE_RANGE.
 * Cache layout of one layer (all device memory, caller-owned, 16-byte aligned):
 *   codes  uint8  [B][Hkv][L_cap][D/2]
 *   params uint32 [B][Hkv][L_cap][D/128]
 * with L_cap % 64 == 0 (the capacity in tokens); K and V have one of each. */
#define BQ_KV4_CAP_MULTIPLE 64

/* Bytes of the codes / params of `rows` cached vectors; -1 if d is not 128 or
 * 256 or rows < 0. */
int64_t bq_kv4_codes_bytes(int64_t rows, int d);
int64_t bq_kv4_params_bytes(int64_t rows, int d);

/* Quantise `rows` contiguous BF16 vectors x [rows][d] into codes [rows][d/2]
 * and params [rows][d/128] (for example one sequence's and KV head's prompt
 * keys, written straight into its cache rows).  All pointers device, 16-byte
 * aligned.  Bit-exact to the definition above.  Asynchronous on `stream`;
 * group errors surface through bq_check(). */
bq_status bq_kv4_quantize(const uint16_t* x, int64_t rows, int d, uint8_t* codes, uint32_t* params,
                          void* stream);

/* Append one decode step: the new key and value of every sequence b and KV
 * head h (k, v BF16 [B][Hkv][d]) are quantised into row pos[b] of their caches
 * (codes / params laid out as above).  pos: device int32 [B]; a position
 * outside [0, L_cap) writes nothing for that sequence and makes bq_check()
 * report BQ_ERR_SHAPE.  Asynchronous on `stream`. */
bq_status bq_kv4_append(const uint16_t* k, const uint16_t* v, int batch, int hkv, int d, const int32_t* pos,
                        int64_t l_cap, uint8_t* k_codes, uint32_t* k_params, uint8_t* v_codes,
                        uint32_t* v_params, void* stream);

/* Workspace bytes bq_kv4_attention_decode needs (0 when the context is not
 * split across CTAs); -1 for an invalid shape. */
int64_t bq_kv4_attention_workspace_bytes(int batch, int hq, int hkv, int d, int64_t l_cap, int64_t max_len);

/* Decode attention over the 4-bit cache, one query token per sequence:
 *   for query head h of sequence b (KV head kv = h / G, G = hq / hkv <= 8) and
 *   its first lens[b] cached tokens t:
 *     a_t = scale <q[b][h], K_t>,  p_t = exp(a_t - max a),
 *     out[b][h] = sum_t p_t V_t / sum_t p_t     (zeros when lens[b] == 0),
 * with K_t, V_t the dequantised cache rows (s c + z).
 * q BF16 [B][hq][d]; out [B][hq][d] BF16 or F32 (out_dtype); lens device int32
 * [B] with 0 <= lens[b] <= max_len <= L_cap (a length outside that range is
 * clamped into it and bq_check() reports BQ_ERR_SHAPE); d 128 or 256;
 * B * hkv <= 65535.  The kernel reads whole stages of 64 (d = 128) or 32
 * tokens, so cache rows up to the next multiple of that past lens[b] are read
 * (never past L_cap) but do not enter the result.
 * Precision: |out - exact| <= 2e-3 * sum_t p_t (|V_tj| + 8 |s_t|) / sum_t p_t
 * (s_t the scale of V_tj's group) plus the output rounding (2^-8 |out| for
 * BF16), while every token's scale * sum_j |q_j K_tj| stays below 256.
 * workspace: >= bq_kv4_attention_workspace_bytes() device bytes, 256-byte
 * aligned, ZERO-FILLED before its first use; every call leaves its counters
 * zero (calls sharing a workspace must not overlap on the GPU; after a
 * BQ_ERR_TIMEOUT zero it again).  The result does not depend on timing (the
 * context splits are merged in a fixed order).  Asynchronous on `stream`. */
bq_status bq_kv4_attention_decode(const uint16_t* q, const uint8_t* k_codes, const uint32_t* k_params,
                                  const uint8_t* v_codes, const uint32_t* v_params, const int32_t* lens,
                                  int batch, int hq, int hkv, int d, int64_t l_cap, int64_t max_len,
                                  float scale, void* out, int out_dtype, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------ errors */
/* Synchronises `stream`, then reports a pending CUDA error (BQ_ERR_CUDA) or a
 * device wait that timed out since the last check (BQ_ERR_TIMEOUT, and the
 * flag is cleared).  BQ_OK otherwise. */
bq_status bq_check(void* stream);
/* Test hook for the time-out path: run one kernel that waits on a flag that
 * nothing sets, with a limit of `spin_limit` polls; it gives up, records
 * BQ_ERR_TIMEOUT and returns.  Never hangs. */
bq_status bq_debug_wait_timeout(int64_t spin_limit, void* stream);
/* Static, NUL-terminated description of a status code. */
const char* bq_status_string(int status);
/* Library version as 10000*major + 100*minor + patch. */
int bq_version(void);

#ifdef __cplusplus
}
#endif
#endif /* BQ_H */
