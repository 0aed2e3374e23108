// Decode GEMV, one launch per call: each CTA owns a contiguous range of whole
// weight rows and reduces over all of K itself, so there is no workspace, no
// preparation kernel and no cross-CTA reduction (binary g128, 2-bit-slot and
// 5-trits-per-byte ternary g128, batch 1..8, K % 1024 == 0, while the
// activation operand of all of K fits in shared memory).
//
// Arithmetic: the codes are expanded with one LOP3 per four weights into int8
// operands of the warp MMA m16n8k32,
//   binary : byte j of (w & (0x01010101 << p)) = 2^p * bit(8j+p),
//   2-bit  : byte j of (w & (0x03030303 << 2i)) = 4^i * c(4j+i), c = q+1,
//   affine : the binary bits, w = s b + z ("Bonsai-27B ... Binary g128", section
//            "MLX打包优化": a scale and a bias per group),
//   5-trit : a byte v = sum c_i 3^i ("把 27B 模型压到 4GB" section 2.4: 3^5 <= 256)
//            gives c0..c3 as the four bytes of a 256-entry table word (one
//            copy per lane in shared memory, so lookups never conflict) and
//            c4 = (810 v) >> 16 (exact for v < 243),
// against activations in per-(batch row, group) fixed point: with 2^E mapping
// the group's largest |x| into [2^29, 2^30), the k-slot of class p (binary) or
// i (2-bit) carries B = round(x 2^(E-p)) resp. round(x 2^(E-2i)), so that the
// product A * B = bit * x * 2^E (resp. c * x * 2^E) up to 2^(p-1) units of
// 2^-E (at most 2^-23 of the group's largest |x| per element).  B is split
// into four signed base-256 digits, one MMA column each.  Per group and row the
// int32 column sums are recombined in FP32:
//   binary : y += s * (2 * 2^-E * sum bit B 2^p - z)
//   ternary: y += s * (    2^-E * sum c   B 4^i - z)
//   affine : y += s * 2^-E * sum bit B 2^p + zb * z   (zb the group's bias)
// with z the group's activation sum in FP32 ("Bonsai-27B ... Binary g128":
// 0 -> -scale, 1 -> +scale; "1-bit Bonsai 8B" notes, section 4.1: one FP16
// scale per 128 weights).
//
// CTA: NW compute warps and one producer warp, in one of two shapes.
//   * NW = 8, at most half of an SM's shared memory and registers, two CTAs
//     per SM: the largest matrices (LM heads) at batch 1-2, where each warp
//     takes two row tiles of a 16-tile chunk and reuses the activation
//     fragments of a group for both.
//   * NW = 16, one CTA per SM: everything else.
//   The producer streams the CTA's weights -- per (chunk of row tiles of 16
//   rows; stage of 1024 K) TMA boxes of codes (128-byte swizzle) and scales --
//   into a ring of shared-memory slots, starting before the wait on the
//   previous kernel in the stream (the weights do not depend on it).  A full
//   chunk is one 128-row box per 128-byte column (one TMA instruction per
//   16 KB); a partial chunk uses 16-row boxes, one lane per tile.
//   After that wait the compute warps turn x into the MMA B fragments and the
//   per-group recombination table for all of K, into shared memory; the work
//   is spread over every compute lane (one lane per 16 activations).
//   A chunk of CT row tiles gives each warp TPW = CT / NW row tiles (CT >= NW)
//   or gives each row tile NW / CT warps, each taking a contiguous share of the
//   stage's 8 groups; the warps sharing a row tile add their partial sums
//   through shared memory in warp order (deterministic).
#include <cuda.h>

#include "bq_internal.cuh"
#include "bq_ptx.cuh"

namespace bq {
namespace rows {

constexpr int kGroupsPerStage = 8;  // 1024 K per stage
constexpr int kMaxChunkTiles = 8;   // chunk bound of the 2-bit and 5-trit formats
constexpr int kTileScaleBytes = 16 * kGroupsPerStage * 2;  // 256: one FP16 scale per group
// The bit formats: binary and affine share the code layout and its decode.
template <int FMT>
constexpr bool bits_fmt() { return FMT == BQ_Q1G128 || FMT == BQ_A1G128; }
// FP16 values per group in the scale plane: the scale, or the (scale, bias)
// pair of the affine format.
template <int FMT>
constexpr int spg() { return FMT == BQ_A1G128 ? 2 : 1; }
template <int FMT>
constexpr int tile_scale_bytes() { return kTileScaleBytes * spg<FMT>(); }
constexpr int kMaxSlots = 8;
constexpr int kSmemFull = 232448;  // opt-in shared memory per block on sm_100 (one CTA per SM)
constexpr int kSmemHalf = 115712;  // two CTAs per SM: (228 KB - 2 x 1 KB reserved) / 2
constexpr uint32_t kWaitPolls = 1u << 23;

template <int NW>
constexpr int threads_of() { return (NW + 1) * 32; }

template <int FMT>
struct Fmt;
template <>
struct Fmt<BQ_Q1G128> {
    static constexpr int kBoxes = 1;      // 128-byte columns per row tile and stage
    static constexpr int kCoefShift = 1;  // 2 * sum(bit * x) - sum(x)
};
template <>
struct Fmt<BQ_A1G128> {
    static constexpr int kBoxes = 1;
    static constexpr int kCoefShift = 0;  // sum(bit * x), the bias term added apart
};
template <>
struct Fmt<BQ_T2G128> {
    static constexpr int kBoxes = 2;
    static constexpr int kCoefShift = 0;  // sum(c * x) - sum(x)
};
template <>
struct Fmt<BQ_T5P8G128> {
    static constexpr int kBoxes = 1;      // one unswizzled 208-byte column (8 groups x 26 bytes)
    static constexpr int kCoefShift = 0;  // sum(c * x) - sum(x)
};
constexpr int kT5RowBytes = kGroupsPerStage * 26;  // 208
constexpr int kLutBytes = 256 * 32 * 4;           // byte -> c0..c3, one copy per lane
// Slot layout: codes [column box b][row tile i][16 rows][128 B] (so that a
// 128-row box of column b lands on 8 row tiles at once; 5-trit format:
// [row tile i][16 rows][208 B]), then scales [row tile i][16 rows][8 groups]
// FP16.
template <int FMT>
constexpr int tile_code_bytes() { return FMT == BQ_T5P8G128 ? 16 * kT5RowBytes : Fmt<FMT>::kBoxes * 16 * 128; }
constexpr int kBoxColumnBytes = kMaxChunkTiles * 16 * 128;  // 16 KB
// Largest chunk (row tiles) a kernel is built for: 16 for the binary format
// up to batch 4 (two row tiles per warp at NW = 8, one at NW = 16), else 8.
template <int FMT, int NT>
constexpr int mct() { return (bits_fmt<FMT>() && NT <= 2) ? 16 : kMaxChunkTiles; }

struct Params {
    const uint16_t* x;  // [batch][K] BF16
    void* y;            // [batch][N]
    int64_t n, k;
    int batch, y_dtype;
    int stages;         // K / 1024
    int row_tiles;      // ceil(N / 16)
    int slots;          // ring slots
    int slot_bytes;     // bytes per slot (chunk_cap row tiles)
    int scales_off;     // offset of the scale tiles within a slot
    int chunk_cap;      // row tiles per chunk, at most; column boxes of 2-bit
                        // codes are chunk_cap * 2 KB apart in a slot
    uint32_t x_off, red_off, lut_off, bar_off;  // shared-memory offsets
    int* status;
    // SwiGLU epilogue (persistent chain kernel only; 0 otherwise): the W rows
    // are [gate; up], a CTA's row tiles are gate tiles paired with the up
    // tiles pair_tiles further on, and y receives BF16(silu(gate) * up)
    int pair_tiles;
    uint32_t stg_off;  // staging of a chunk's sums for that epilogue
};

// Position in the slot ring (the ring depth is a runtime value: no divisions).
struct Ring {
    int slot = 0, depth = 1;
    uint32_t round = 0;  // times the ring has wrapped
    __device__ __forceinline__ void next() {
        if (++slot == depth) {
            slot = 0;
            ++round;
        }
    }
};

template <int NW>
__device__ __forceinline__ void bar_compute() { asm volatile("bar.sync 1, %0;" ::"n"(NW * 32) : "memory"); }

// A chunk takes as many of the remaining tiles as the cap allows (any count);
// it runs in the compiled shape of the next power of two, the tiles past its
// count idle (one pass over K for, e.g., three tiles instead of a pass for two
// and one for one).
__device__ __forceinline__ int chunk_count(int remaining, int cap) { return remaining < cap ? remaining : cap; }

// Bytes of the resident activation operand per (stage, n-tile): B fragments
// [8 groups][2 MMA pairs][LANES][16 B] then the table [8 groups][4][float4].
__host__ __device__ constexpr int x_nt_bytes(int lanes) { return kGroupsPerStage * 2 * lanes * 16 + kGroupsPerStage * 4 * 16; }

// 2^e as a float, e in [-126, 127].
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((e + 127) << 23); }

// floor(log2 m) for a finite m > 0, subnormals included.
__device__ __forceinline__ int ilog2f(float m) {
    const int b = __float_as_int(m);
    const int ex = (b >> 23) & 0xFF;
    return ex ? ex - 127 : (31 - __clz(b & 0x7FFFFF)) - 149;
}

// ------------------------------------------------------------ activation prep
// The byte of digit d of batch row bb for weight k goes to the
// B fragment of lane (4 (d + 4 (bb & 1)) + t), MMA q, register h, byte j,
// where (t, q, h, j) is the k-slot the A decode gives weight k:
//   binary: k = 32t + 8j + 2q + h   (word t of the row's group, class 2q+h)
//   2-bit : k = 32t + 16h + 4j + q  (word 2t+h of the row's group, class q)
//   5-trit: A register i = 2q + h of thread t holds, for i < 6, digits 0..3
//           of byte 6t+i; i = 6 digit 4 of bytes 6t..6t+3; i = 7 digit 4 of
//           bytes 6t+4, 6t+5 and trits 120+2t, 121+2t (the group's last
//           eight trits, in bytes 24 and 25)
// Table entry (G, t) of an n-tile, t = 2 (bb & 1) + hh for digit pair hh, with
// e = coef - E + 16 hh and z = [hh == 0] times the group's activation sum:
//   one factor  : {2^e, 1, z, 0}, u = (D0 + 256 D1) 2^e - z;
//   two factors : {2^a, 2^(e-a), z, 1} when 2^e is not a normal float,
//                 u = (D0 + 256 D1) 2^a 2^(e-a) - z.
// Rows past the batch are prepared as zero activations (zero digits, z = 0).
//
// Work split: a task is (group G, B-fragment thread t, MMA pair P) of one
// stage and batch row: the 16 activations that land in pair P of thread t's
// slots.  Byte 4 m + j of the 16-byte chunk (pair P, digit d) is digit d of
// activation prep_src(P, m, j) of the thread's 32 (k = 32 t + r for binary
// and 2-bit; k = 30 t + r, r < 30, and 120 + 2 t + (r - 30) for 5-trit), so a
// lane assembles its four chunks in registers (a 4 x 4 byte transpose per m)
// and stores them whole.  Lane 8 g + 2 t + P of a warp takes group 4 h + g of
// half h of a stage; the group's eight lanes share the maximum and the sum
// through shuffles.
template <int FMT>
__device__ __forceinline__ constexpr int prep_src(int P, int m, int j) {
    if (bits_fmt<FMT>()) return 8 * j + 4 * P + m;                        // k = 32t + 8j + 2q + h
    if (FMT == BQ_T2G128) return 16 * (m & 1) + 4 * j + 2 * P + (m >> 1);  // k = 32t + 16h + 4j + q
    if (P == 0) return 5 * m + j;                 // digits 0..3 of bytes 6t .. 6t+3
    if (m < 2) return 20 + 5 * m + j;             // digits 0..3 of bytes 6t+4, 6t+5
    if (m == 2) return 5 * j + 4;                 // digit 4 of bytes 6t .. 6t+3
    return j == 0 ? 24 : j == 1 ? 29 : 28 + j;    // digit 4 of 6t+4, 6t+5; trits 120+2t, 121+2t
}

// Class of activation (P, m, j) as a left shift: the operand's power of two
// (binary: the bit's weight 2^class; 2-bit: 4^class).
template <int FMT>
__device__ __forceinline__ int prep_class_shift(int P, int m) {
    if (bits_fmt<FMT>()) return 4 * P + m;               // (8j + 4P + m) mod 8
    if (FMT == BQ_T2G128) return 2 * (2 * P + (m >> 1));  // 2 * ((16(m&1) + 4j + 2P + (m>>1)) mod 4)
    return 0;
}

// The task's activations.  Binary: the four runs k = 32t + 8j + 4P + {0..3}
// (value 4j + m of raw); 2-bit: the pairs k = 32t + 4j + 2P + {0,1} and
// 32t + 16 + 4j + 2P + {0,1} (words 2j and 2j + 1 of raw); 5-trit: all 32
// activations of thread t (value r of raw, both pairs).  xg is the group's
// first activation (16-byte aligned).  COHERENT: the loads go through L2 (the
// chain kernel, where x may have been written by other CTAs of the same
// launch); otherwise through the non-coherent cached path.
template <bool COHERENT, typename T>
__device__ __forceinline__ T ld_x(const T* p) { return COHERENT ? __ldcg(p) : __ldg(p); }

template <int FMT, bool COHERENT>
__device__ __forceinline__ void load_task_x(const uint16_t* xg, int t, int P, uint32_t (&raw)[16]) {
    if (bits_fmt<FMT>()) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint2 v = ld_x<COHERENT>(reinterpret_cast<const uint2*>(xg + 32 * t + 8 * j + 4 * P));
            raw[2 * j] = v.x;
            raw[2 * j + 1] = v.y;
        }
    } else if (FMT == BQ_T2G128) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            raw[2 * j] = ld_x<COHERENT>(reinterpret_cast<const uint32_t*>(xg + 32 * t + 4 * j + 2 * P));
            raw[2 * j + 1] = ld_x<COHERENT>(reinterpret_cast<const uint32_t*>(xg + 32 * t + 16 + 4 * j + 2 * P));
        }
    } else {
        const uint32_t* src = reinterpret_cast<const uint32_t*>(xg + 30 * t);  // 60 t bytes: 4-byte aligned
#pragma unroll
        for (int i = 0; i < 15; ++i) raw[i] = ld_x<COHERENT>(src + i);
        raw[15] = ld_x<COHERENT>(reinterpret_cast<const uint32_t*>(xg + 120 + 2 * t));
    }
}

__device__ __forceinline__ float raw_value(const uint32_t (&raw)[16], int r) {
    return __uint_as_float((r & 1) ? (raw[r >> 1] & 0xFFFF0000u) : (raw[r >> 1] << 16));
}

// Activation (P, m, j) of the task (see load_task_x).
template <int FMT>
__device__ __forceinline__ float task_value(const uint32_t (&raw)[16], int P, int m, int j) {
    if (bits_fmt<FMT>()) return raw_value(raw, 4 * j + m);
    if (FMT == BQ_T2G128) return raw_value(raw, 2 * (2 * j + (m & 1)) + (m >> 1));
    const float v0 = raw_value(raw, prep_src<FMT>(0, m, j)), v1 = raw_value(raw, prep_src<FMT>(1, m, j));
    return P ? v1 : v0;
}

// Rows 0 .. 3 of a 4 x 4 byte matrix given as rows a, b, c, e, returned as
// its columns: out[d] = {a.d, b.d, c.d, e.d}.
__device__ __forceinline__ void transpose_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t e, uint32_t (&out)[4]) {
    const uint32_t ab_lo = __byte_perm(a, b, 0x5140), ab_hi = __byte_perm(a, b, 0x7362);
    const uint32_t ce_lo = __byte_perm(c, e, 0x5140), ce_hi = __byte_perm(c, e, 0x7362);
    out[0] = __byte_perm(ab_lo, ce_lo, 0x5410);
    out[1] = __byte_perm(ab_lo, ce_lo, 0x7632);
    out[2] = __byte_perm(ab_hi, ce_hi, 0x5410);
    out[3] = __byte_perm(ab_hi, ce_hi, 0x7632);
}

// One lane's task (group G, thread t, pair P, batch row parity hb of the
// n-tile at xt): its four B-fragment chunks and, on P = 0, t < 2, the table
// entry of digit pair t.  All eight lanes of the group run it together
// (shuffles).
template <int FMT, int LANES>
__device__ __forceinline__ void prep_task(uint8_t* xt, int G, int t, int P, int hb, const uint32_t (&raw)[16]) {
    // group maximum of |x| on the BF16 bits (a larger magnitude has larger bits)
    constexpr int kWords = FMT == BQ_T5P8G128 ? 16 : 8;
    uint32_t mx = 0;
#pragma unroll
    for (int i = 0; i < kWords; ++i) mx = __vmaxu2(mx, raw[i] & 0x7FFF7FFFu);
    mx = max(mx & 0xFFFFu, mx >> 16);
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
    const float m = __uint_as_float(mx << 16);
    const int E = (m > 0.f) ? 29 - ilog2f(m) : 0;  // in [-98, 162]
    // operand multipliers 2^(E - class): one factor unless 2^E leaves the
    // normal range (largest |x| below ~2^-97), then 2^(E-127) * 2^(127-class)
    const bool two = E > 127;
    const float pa = exp2i(two ? E - 127 : 0);
    const int Eb = two ? 127 : E;
    float mul[4];
#pragma unroll
    for (int mm = 0; mm < 4; ++mm) mul[mm] = exp2i(Eb - prep_class_shift<FMT>(P, mm));
    const bool any_two = __any_sync(0xffffffffu, two);
    float zs = 0.0f;
    uint32_t col[4][4];  // [m][digit]
#pragma unroll
    for (int mm = 0; mm < 4; ++mm) {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float v = task_value<FMT>(raw, P, mm, j);
            zs += v;
            const int b = __float2int_rn(any_two ? (v * pa) * mul[mm] : v * mul[mm]);
            // balanced base-256 digits of b (|b| <= 2^30) are the bytes of
            // (b + 0x808080) ^ 0x808080 (the xor is applied after the transpose)
            w[j] = (uint32_t)b + 0x808080u;
        }
        transpose_bytes(w[0], w[1], w[2], w[3], col[mm]);
    }
    uint8_t* xb = xt + ((G * 2 + P) * LANES + 16 * hb + t) * 16;  // chunk (P, digit 0)
#pragma unroll
    for (int d = 0; d < 4; ++d) {
        const uint32_t f = d < 3 ? 0x80808080u : 0u;
        *reinterpret_cast<uint4*>(xb + 4 * d * 16) =
            make_uint4(col[0][d] ^ f, col[1][d] ^ f, col[2][d] ^ f, col[3][d] ^ f);
    }
    // z = the group's activation sum (FP32, fixed order: each lane's 16 in
    // order, then pairs of lanes by xor 1, 2, 4)
    zs += __shfl_xor_sync(0xffffffffu, zs, 1);
    zs += __shfl_xor_sync(0xffffffffu, zs, 2);
    zs += __shfl_xor_sync(0xffffffffu, zs, 4);
    if (P == 0 && t < 2) {
        const int hh = t;  // digit pair (0,1) or (2,3)
        const int e = Fmt<FMT>::kCoefShift - E + 16 * hh;
        const bool tf = Fmt<FMT>::kCoefShift - E < -126;
        const int a = tf ? max(-60, min(60, e)) : e;
        float4* tabp = reinterpret_cast<float4*>(xt + kGroupsPerStage * 2 * LANES * 16) + G * 4 + 2 * hb + hh;
        *tabp = make_float4(exp2i(a), exp2i(e - a), hh == 0 ? zs : 0.0f, tf ? 1.0f : 0.0f);
    }
}

// ------------------------------------------------------------ 5-trit decode
// The 8 A registers of one row of a 5-trit group for thread t (see the
// mapping above).  p: the group's 26 bytes in shared memory; lut: the table
// (word of byte v for lane l at lut[32 v + l]); sel: byte selector of lane t.
__device__ __forceinline__ uint32_t lds_u16(const uint8_t* p) { return *reinterpret_cast<const uint16_t*>(p); }

__device__ __forceinline__ void t5_row(const uint8_t* p, const uint32_t* lut, int t, int lane, uint32_t sel,
                                       uint32_t (&R)[8]) {
    const uint32_t u0 = lds_u16(p + 6 * t), u1 = lds_u16(p + 6 * t + 2), u2 = lds_u16(p + 6 * t + 4);
    const uint32_t ue = lds_u16(p + 24);
    const uint32_t v[6] = {u0 & 0xFFu, u0 >> 8, u1 & 0xFFu, u1 >> 8, u2 & 0xFFu, u2 >> 8};
    uint32_t c4[6];
#pragma unroll
    for (int i = 0; i < 6; ++i) {
        R[i] = lut[v[i] * 32 + lane];
        c4[i] = (v[i] * 810u) >> 16;
    }
    const uint32_t b24 = ue & 0xFFu, b25 = ue >> 8;
    const uint32_t e24 = lut[b24 * 32 + lane], e25 = lut[b25 * 32 + lane];
    // bytes 0..7 = trits 120..127: b24 digits 0..3, b24 digit 4, b25 digits 0..2
    const uint32_t hi = ((b24 * 810u) >> 16) | (e25 << 8);
    const uint32_t x01 = __byte_perm(e24, hi, sel);
    R[6] = c4[0] | (c4[1] << 8) | (c4[2] << 16) | (c4[3] << 24);
    R[7] = c4[4] | (c4[5] << 8) | (x01 << 16);
}

// GPW consecutive FP16 scales (the warp's groups of one row and stage) as
// packed pairs; N = 2 * GPW values for the (scale, bias) pairs of the affine
// format.
template <int N>
__device__ __forceinline__ void load_scales(const uint8_t* p, uint32_t (&s)[(N + 1) / 2]) {
    if constexpr (N == 16) {
        const uint4 v0 = *reinterpret_cast<const uint4*>(p), v1 = *reinterpret_cast<const uint4*>(p + 16);
        s[0] = v0.x; s[1] = v0.y; s[2] = v0.z; s[3] = v0.w;
        s[4] = v1.x; s[5] = v1.y; s[6] = v1.z; s[7] = v1.w;
    } else if constexpr (N == 8) {
        const uint4 v = *reinterpret_cast<const uint4*>(p);
        s[0] = v.x; s[1] = v.y; s[2] = v.z; s[3] = v.w;
    } else if constexpr (N == 4) {
        const uint2 v = *reinterpret_cast<const uint2*>(p);
        s[0] = v.x; s[1] = v.y;
    } else if constexpr (N == 2) {
        s[0] = *reinterpret_cast<const uint32_t*>(p);
    } else {
        s[0] = *reinterpret_cast<const uint16_t*>(p);
    }
}

__device__ __forceinline__ float scale_of(const uint32_t* s, int i) {
    return __half2float(__ushort_as_half((uint16_t)((i & 1) ? (s[i >> 1] >> 16) : (s[i >> 1] & 0xFFFFu))));
}

// ------------------------------------------------------------ one chunk
// CT row tiles (16 rows each) starting at row tile rt, all stages.
//   CT >= NW: warp w takes row tiles w + NW i (i < TPW = CT / NW), all groups;
//   CT <  NW: warp w takes row tile w / WPR (WPR = NW / CT warps per row tile,
//             at most 8; warps past CT row tiles only keep the stage barriers
//             going) and the GPW = 8 / WPR groups G = GPW (w % WPR) + i.
template <int FMT, int NT, int LANES, int NW, int CT>
__device__ bool run_chunk(const Params& p, uint8_t* smem, uint64_t* full, uint64_t* empty, int rt, Ring& rp,
                          int warp, int lane, int ct) {
    constexpr int TPW = CT >= NW ? CT / NW : 1;
    constexpr int WPR = CT >= NW ? 1 : ((NW / CT) < kGroupsPerStage ? (NW / CT) : kGroupsPerStage);
    constexpr int GPW = kGroupsPerStage / WPR;  // groups per warp and stage
    constexpr int TCB = tile_code_bytes<FMT>();
    constexpr int TSTRIDE = FMT == BQ_T5P8G128 ? TCB : 2048;  // code bytes between row tiles of a column box
    constexpr int X_NT = x_nt_bytes(LANES);
    const int my_rt = CT >= NW ? warp : warp / WPR;
    const int gsub = CT >= NW ? 0 : warp % WPR;
    // the chunk holds ct <= CT tiles; a warp whose tiles are all past ct idles
    // (with several tiles per warp, the ones past ct are computed on stale
    // slot contents and never stored)
    const bool active = my_rt < ct;
    const int g = lane >> 2, t = lane & 3;
    // at batch 1 the upper 16 lanes (columns of a second batch row) read the
    // lower lanes' fragments: their sums are never stored
    const int blane = lane & (LANES - 1);
    const uint8_t* xres = smem + p.x_off;
    const uint32_t* lut = reinterpret_cast<const uint32_t*>(smem + p.lut_off);
    const uint32_t t5sel = (uint32_t)(2 * t) | ((uint32_t)(2 * t + 1) << 4);
    float yacc[TPW][NT][2];
#pragma unroll
    for (int tp = 0; tp < TPW; ++tp)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) yacc[tp][nt][0] = yacc[tp][nt][1] = 0.0f;
    // this warp's GPW groups of stage st (ring slot `slot`), added into yacc
    auto stage = [&](int st, int slot) {
        const uint8_t* sb = smem + slot * p.slot_bytes;
        const uint8_t* xs = xres + (size_t)st * NT * X_NT;
        constexpr int SN = GPW * spg<FMT>();  // FP16 values of the warp's groups per row
        uint32_t sc[TPW][2][(SN + 1) / 2];
#pragma unroll
        for (int tp = 0; tp < TPW; ++tp) {
            const uint8_t* srow =
                sb + p.scales_off + (my_rt + NW * tp) * tile_scale_bytes<FMT>() + gsub * GPW * 2 * spg<FMT>();
            load_scales<SN>(srow + g * 16 * spg<FMT>(), sc[tp][0]);
            load_scales<SN>(srow + (g + 8) * 16 * spg<FMT>(), sc[tp][1]);
        }
#pragma unroll
        for (int gi = 0; gi < GPW; ++gi) {
            const int G = gsub * GPW + gi;
            uint4 bf[NT][2];
            float4 tab[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const uint8_t* xt = xs + nt * X_NT;
#pragma unroll
                for (int h = 0; h < 2; ++h) bf[nt][h] = *reinterpret_cast<const uint4*>(xt + ((G * 2 + h) * LANES + blane) * 16);
                tab[nt] = *reinterpret_cast<const float4*>(xt + kGroupsPerStage * 2 * LANES * 16 + (G * 4 + t) * 16);
            }
#pragma unroll
            for (int tp = 0; tp < TPW; ++tp) {
                const uint8_t* codes_t = sb + (my_rt + NW * tp) * TSTRIDE;  // column box 0 of this row tile
                int acc[NT][4];
                if (bits_fmt<FMT>()) {
                    const int off = ((G ^ g) << 4) + 4 * t;
                    const uint32_t w0 = *reinterpret_cast<const uint32_t*>(codes_t + g * 128 + off);
                    const uint32_t w1 = *reinterpret_cast<const uint32_t*>(codes_t + (g + 8) * 128 + off);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t m0 = 0x01010101u << (2 * q), m1 = 0x01010101u << (2 * q + 1);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const uint32_t b0 = (q & 1) ? bf[nt][q >> 1].z : bf[nt][q >> 1].x;
                            const uint32_t b1 = (q & 1) ? bf[nt][q >> 1].w : bf[nt][q >> 1].y;
                            if (q == 0)
                                ptx::mma_u8s8_init(acc[nt], w0 & m0, w1 & m0, w0 & m1, w1 & m1, b0, b1, 0);
                            else
                                ptx::mma_u8s8(acc[nt], w0 & m0, w1 & m0, w0 & m1, w1 & m1, b0, b1);
                        }
                    }
                } else if (FMT == BQ_T5P8G128) {
                    const uint8_t* g0 = codes_t + g * kT5RowBytes + 26 * G;
                    uint32_t R0[8], R1[8];
                    t5_row(g0, lut, t, lane, t5sel, R0);
                    t5_row(g0 + 8 * kT5RowBytes, lut, t, lane, t5sel, R1);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const uint32_t b0 = (q & 1) ? bf[nt][q >> 1].z : bf[nt][q >> 1].x;
                            const uint32_t b1 = (q & 1) ? bf[nt][q >> 1].w : bf[nt][q >> 1].y;
                            if (q == 0)
                                ptx::mma_u8s8_init(acc[nt], R0[0], R1[0], R0[1], R1[1], b0, b1, 0);
                            else
                                ptx::mma_u8s8(acc[nt], R0[2 * q], R1[2 * q], R0[2 * q + 1], R1[2 * q + 1], b0, b1);
                        }
                    }
                } else {
                    // words 2t, 2t+1 of the row's 32-byte group
                    const uint8_t* box = codes_t + (G >> 2) * (p.chunk_cap * 2048);  // column box 1 after chunk_cap tiles
                    const int chunk = 2 * (G & 3) + (t >> 1);
                    const int off = ((chunk ^ g) << 4) + 8 * (t & 1);
                    const uint2 wr0 = *reinterpret_cast<const uint2*>(box + g * 128 + off);
                    const uint2 wr1 = *reinterpret_cast<const uint2*>(box + (g + 8) * 128 + off);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t m = 0x03030303u << (2 * q);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const uint32_t b0 = (q & 1) ? bf[nt][q >> 1].z : bf[nt][q >> 1].x;
                            const uint32_t b1 = (q & 1) ? bf[nt][q >> 1].w : bf[nt][q >> 1].y;
                            if (q == 0)
                                ptx::mma_u8s8_init(acc[nt], wr0.x & m, wr1.x & m, wr0.y & m, wr1.y & m, b0, b1, 0);
                            else
                                ptx::mma_u8s8(acc[nt], wr0.x & m, wr1.x & m, wr0.y & m, wr1.y & m, b0, b1);
                        }
                    }
                }
                const float s0 = scale_of(sc[tp][0], spg<FMT>() * gi), s1 = scale_of(sc[tp][1], spg<FMT>() * gi);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    // D0 + 256 D1 is exact in int32 (|D0|, |D1| <= 2^21)
                    const float v0 = (float)(acc[nt][0] + (acc[nt][1] << 8));
                    const float v1 = (float)(acc[nt][2] + (acc[nt][3] << 8));
                    if constexpr (FMT == BQ_A1G128) {
                        // s * sum(bit x) + zb * sum(x) (the sum on digit pair 0 only)
                        const float z0 = scale_of(sc[tp][0], 2 * gi + 1), z1 = scale_of(sc[tp][1], 2 * gi + 1);
                        yacc[tp][nt][0] = fmaf(s0, v0 * tab[nt].x * tab[nt].y, fmaf(z0, tab[nt].z, yacc[tp][nt][0]));
                        yacc[tp][nt][1] = fmaf(s1, v1 * tab[nt].x * tab[nt].y, fmaf(z1, tab[nt].z, yacc[tp][nt][1]));
                    } else {
                        // (with one factor tab.y = 1: the same rounding as fmaf(v, 2^e, -z))
                        const float u0 = fmaf(v0 * tab[nt].x, tab[nt].y, -tab[nt].z);
                        const float u1 = fmaf(v1 * tab[nt].x, tab[nt].y, -tab[nt].z);
                        yacc[tp][nt][0] = fmaf(s0, u0, yacc[tp][nt][0]);
                        yacc[tp][nt][1] = fmaf(s1, u1, yacc[tp][nt][1]);
                    }
                }
            }
        }
    };
    // Binary format: where a warp has fewer than four (group, n-tile) pairs per
    // stage, stages are taken U at a time, so that U independent MMA chains run
    // between two barrier waits, if the ring holds 2 U slots.  (The longer
    // 2-bit and 5-trit stage bodies measured slower this way.)
    constexpr int U = (!bits_fmt<FMT>() || GPW * NT * TPW >= 4) ? 1 : 4 / (GPW * NT * TPW);
    const int ustep = (U > 1 && p.slots >= 2 * U) ? U : 1;  // (the producer keeps U slots ahead)
    bool alive = true;
    for (int st = 0; st < p.stages; st += ustep) {
        const int nst = min(ustep, p.stages - st);
        const Ring r0 = rp;  // ring position of stage st
        int su[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            su[u] = rp.slot;
            if (u < nst && alive) {
                if (!ptx::mbar_wait_bounded(&full[rp.slot], rp.round & 1u, kWaitPolls)) {
                    record_status(p.status, BQ_ERR_TIMEOUT);
                    alive = false;
                }
                rp.next();
            }
        }
        if (!alive) break;
        if (active) {
            if constexpr (U == 1) {
                stage(st, su[0]);
            } else if (nst == U) {
#pragma unroll
                for (int u = 0; u < U; ++u) stage(st + u, su[u]);
            } else {
                // (tail, or a ring too shallow for U: one stage at a time)
                Ring rs = r0;
#pragma unroll 1
                for (int u = 0; u < nst; ++u, rs.next()) stage(st + u, rs.slot);
            }
        }
        __syncwarp();
        if (lane == 0) {
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (u < nst) ptx::mbar_arrive(&empty[su[u]]);
        }
    }
    // digit pairs (t, t^1) -> one value per (batch row, row) on even t
#pragma unroll
    for (int tp = 0; tp < TPW; ++tp)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int r = 0; r < 2; ++r) yacc[tp][nt][r] += __shfl_xor_sync(0xffffffffu, yacc[tp][nt][r], 1);
    if (WPR > 1) {
        // partial sums of the warps sharing a row tile, added in warp order
        float* red = reinterpret_cast<float*>(smem + p.red_off);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int r = 0; r < 2; ++r) red[((warp * 32 + lane) * NT + nt) * 2 + r] = yacc[0][nt][r];
        bar_compute<NW>();
        if (active && gsub == 0) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    float s = 0.0f;
#pragma unroll
                    for (int j = 0; j < WPR; ++j) s += red[(((warp + j) * 32 + lane) * NT + nt) * 2 + r];
                    yacc[0][nt][r] = s;
                }
        }
        bar_compute<NW>();  // red is reused by the next chunk
    }
    if (active && gsub == 0 && (t & 1) == 0 && p.pair_tiles > 0) {
        // SwiGLU step: the chunk's sums go to the staging area [tile][row][batch]
        float* stg = reinterpret_cast<float*>(smem + p.stg_off);
#pragma unroll
        for (int tp = 0; tp < TPW; ++tp)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int r = 0; r < 2; ++r)
                    if (my_rt + NW * tp < ct)
                        stg[((my_rt + NW * tp) * 16 + g + 8 * r) * 8 + nt * 2 + (t >> 1)] = yacc[tp][nt][r];
    } else if (active && gsub == 0 && (t & 1) == 0) {
#pragma unroll
        for (int tp = 0; tp < TPW; ++tp)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int bb = nt * 2 + (t >> 1);
                    const int64_t row = (int64_t)(rt + my_rt + NW * tp) * 16 + g + 8 * r;
                    if (bb < p.batch && row < p.n && my_rt + NW * tp < ct) {
                        if (p.y_dtype == BQ_F32)
                            static_cast<float*>(p.y)[bb * p.n + row] = yacc[tp][nt][r];
                        else
                            static_cast<uint16_t*>(p.y)[bb * p.n + row] = float_to_bf16_bits(yacc[tp][nt][r]);
                    }
                }
    }
    return alive;
}

// ------------------------------------------------------------ kernel
// Tensor maps: codes and scales with 16-row boxes (partial chunks) and
// 128-row boxes (full chunks).
struct Maps {
    CUtensorMap codes16, scales16, codes128, scales128;
};

// Row tile of W that tile i of a chunk of ct tiles starting at r holds: r + i,
// or, for a SwiGLU step, gate tiles r .. r + ct/2 - 1 then the up tiles
// pair_tiles further on.
__device__ __forceinline__ int chunk_row_tile(const Params& p, int r, int ct, int i) {
    if (p.pair_tiles == 0) return r + i;
    const int c = ct >> 1;
    return i < c ? r + i : p.pair_tiles + r + (i - c);
}

// The producer's copies of one (chunk, stage) into ring slot `slot`; lane 0
// has posted the byte count on full[slot].  A full chunk is one 128-row box per
// 128-byte column and 8 row tiles whose rows are contiguous; otherwise 16-row
// boxes, one lane per row tile.
template <int FMT>
__device__ __forceinline__ void issue_stage(const Maps& tm, const Params& p, uint8_t* smem, uint64_t* full, int slot,
                                            int st, int r, int ct, int lane) {
    constexpr int TCB = tile_code_bytes<FMT>();
    constexpr int KB = Fmt<FMT>::kBoxes;
    uint8_t* sb = smem + slot * p.slot_bytes;
    const bool box128 = FMT == BQ_T5P8G128
                            ? (ct == kMaxChunkTiles && p.pair_tiles == 0)
                            : (ct % kMaxChunkTiles == 0 && (p.pair_tiles == 0 || ct >= 2 * kMaxChunkTiles));
    if (FMT == BQ_T5P8G128) {
        if (box128) {
            if (lane == 0) ptx::tma_load_2d(sb, &tm.codes128, st * kT5RowBytes, r * 16, &full[slot]);
            if (lane == 1)
                ptx::tma_load_2d(sb + p.scales_off, &tm.scales128, st * kGroupsPerStage, r * 16, &full[slot]);
        } else if (lane < ct) {
            const int rt = chunk_row_tile(p, r, ct, lane);
            ptx::tma_load_2d(sb + lane * TCB, &tm.codes16, st * kT5RowBytes, rt * 16, &full[slot]);
            ptx::tma_load_2d(sb + p.scales_off + lane * kTileScaleBytes, &tm.scales16, st * kGroupsPerStage, rt * 16,
                             &full[slot]);
        }
    } else if (box128) {
        // 128-row boxes: one per 128-byte column (2-bit) and 8 row tiles
        const int nbox = ct / kMaxChunkTiles;
        if (lane < nbox * KB) {
            const int h8 = lane / KB, b = lane - h8 * KB;
            ptx::tma_load_2d(sb + b * (p.chunk_cap * 2048) + h8 * kBoxColumnBytes, &tm.codes128,
                             st * (KB * 128) + b * 128, chunk_row_tile(p, r, ct, 8 * h8) * 16, &full[slot]);
        } else if (lane >= 16 && lane < 16 + nbox) {
            const int h8 = lane - 16;
            ptx::tma_load_2d(sb + p.scales_off + h8 * kMaxChunkTiles * tile_scale_bytes<FMT>(), &tm.scales128,
                             st * kGroupsPerStage * spg<FMT>(), chunk_row_tile(p, r, ct, 8 * h8) * 16, &full[slot]);
        }
    } else if (lane < ct) {
        const int rt = chunk_row_tile(p, r, ct, lane);
#pragma unroll
        for (int b = 0; b < KB; ++b)
            ptx::tma_load_2d(sb + b * (p.chunk_cap * 2048) + lane * 2048, &tm.codes16, st * (KB * 128) + b * 128,
                             rt * 16, &full[slot]);
        ptx::tma_load_2d(sb + p.scales_off + lane * tile_scale_bytes<FMT>(), &tm.scales16,
                         st * kGroupsPerStage * spg<FMT>(), rt * 16, &full[slot]);
    }
}

// Producer warp: streams the weights of row tiles [rt0, rt1) (pair tiles for
// a SwiGLU step), chunk by chunk and stage by stage, through the ring.  rp and
// it (copies issued) carry over from one call to the next.  False if a slot
// wait timed out.
template <int FMT>
__device__ __forceinline__ bool produce(const Maps& tm, const Params& p, uint8_t* smem, uint64_t* full, uint64_t* empty, int rt0,
                        int rt1, Ring& rp, int& it, int lane) {
    constexpr int TCB = tile_code_bytes<FMT>();
    const int cap = p.pair_tiles > 0 ? p.chunk_cap / 2 : p.chunk_cap;
    for (int r = rt0; r < rt1;) {
        const int c = chunk_count(rt1 - r, cap);  // the consumer's chunks
        const int ct = p.pair_tiles > 0 ? 2 * c : c;
        for (int st = 0; st < p.stages; ++st, ++it, rp.next()) {
            const int slot = rp.slot;
            int ok = 1;
            if (lane == 0) {
                if (rp.round > 0 && !ptx::mbar_wait_bounded(&empty[slot], (rp.round - 1) & 1u, kWaitPolls)) {
                    record_status(p.status, BQ_ERR_TIMEOUT);
                    ok = 0;
                } else {
                    ptx::mbar_arrive_expect_tx(&full[slot], (uint32_t)(ct * (TCB + tile_scale_bytes<FMT>())));
                }
            }
            if (!__shfl_sync(0xffffffffu, ok, 0)) return false;
            issue_stage<FMT>(tm, p, smem, full, slot, st, r, ct, lane);
        }
        r += c;
    }
    return true;
}

// Compute warps: x -> the resident activation operand (B fragments and table
// of all of K).  Warp items (stage, batch row, half h of the stage's groups),
// item i on warp i % NW; lane 8 gq + 2 t + P takes group 4 h + gq.  Rows go up
// to the n-tiles' width (zero past the batch; one row at 16 lanes).
template <int FMT, int NT, int LANES, int NW, bool COHERENT>
__device__ __forceinline__ void prep_x(const Params& p, uint8_t* smem, int warp, int lane) {
    constexpr int kPrepBatch = 2;
    uint8_t* xres = smem + p.x_off;
    const int rows = LANES == 16 ? 1 : 2 * NT;
    const int items = p.stages * rows * 2;
    const int gq = lane >> 3, t = (lane >> 1) & 3, P = lane & 1;
    for (int i0 = warp; i0 < items; i0 += NW * kPrepBatch) {
        uint32_t raw[kPrepBatch][16];
#pragma unroll
        for (int j = 0; j < kPrepBatch; ++j) {
            const int i = i0 + j * NW;
            const int sr = i >> 1, G = 4 * (i & 1) + gq;
            const int st = sr / rows, bb = sr - st * rows;
            if (i < items && bb < p.batch) {
                load_task_x<FMT, COHERENT>(p.x + (int64_t)bb * p.k + (int64_t)st * 1024 + G * 128, t, P, raw[j]);
            } else {
#pragma unroll
                for (int w = 0; w < 16; ++w) raw[j][w] = 0u;
            }
        }
#pragma unroll
        for (int j = 0; j < kPrepBatch; ++j) {
            const int i = i0 + j * NW;
            if (i < items) {  // (warp-uniform)
                const int sr = i >> 1, G = 4 * (i & 1) + gq;
                const int st = sr / rows, bb = sr - st * rows;
                prep_task<FMT, LANES>(xres + (size_t)(st * NT + (bb >> 1)) * x_nt_bytes(LANES), G, t, P, bb & 1,
                                      raw[j]);
            }
        }
    }
}

// One chunk of ct row tiles in the compiled shape of the next power of two
// (only the shapes up to CAP are compiled in).
template <int FMT, int NT, int LANES, int NW, int CAP>
__device__ __forceinline__ bool chunk_by_size(int ct, const Params& p, uint8_t* smem, uint64_t* full, uint64_t* empty,
                                              int r, Ring& rp, int warp, int lane) {
    if constexpr (CAP >= 16 && mct<FMT, NT>() >= 16) {
        if (ct > 8) return run_chunk<FMT, NT, LANES, NW, mct<FMT, NT>()>(p, smem, full, empty, r, rp, warp, lane, ct);
    }
    if constexpr (CAP >= 8) {
        if (ct > 4) return run_chunk<FMT, NT, LANES, NW, 8>(p, smem, full, empty, r, rp, warp, lane, ct);
    }
    if constexpr (CAP >= 4) {
        if (ct > 2) return run_chunk<FMT, NT, LANES, NW, 4>(p, smem, full, empty, r, rp, warp, lane, ct);
    }
    if (ct == 2) return run_chunk<FMT, NT, LANES, NW, 2>(p, smem, full, empty, r, rp, warp, lane, ct);
    return run_chunk<FMT, NT, LANES, NW, 1>(p, smem, full, empty, r, rp, warp, lane, ct);
}

// Compute warps: every chunk of row tiles [rt0, rt1) (pair tiles for a SwiGLU
// step, whose chunks hold c gate and c up tiles and end with the SwiGLU
// epilogue).  CAP: the largest chunk the launch uses; only the chunk shapes up
// to it are compiled into the kernel (a small matrix's kernel then carries
// the code of its own shapes alone: measured 0.4-0.6 us faster per small call
// than with every shape's code).  False if a wait timed out.
template <int FMT, int NT, int LANES, int NW, int CAP = 16>
__device__ __forceinline__ bool run_chunks(const Params& p, uint8_t* smem, uint64_t* full, uint64_t* empty, int rt0, int rt1,
                           Ring& rp, int warp, int lane) {
    const int cap = p.pair_tiles > 0 ? p.chunk_cap / 2 : p.chunk_cap;
    for (int r = rt0; r < rt1;) {
        const int c = chunk_count(rt1 - r, cap);
        const int ct = p.pair_tiles > 0 ? 2 * c : c;
        const bool ok = chunk_by_size<FMT, NT, LANES, NW, CAP>(ct, p, smem, full, empty, r, rp, warp, lane);
        if (!ok) return false;
        if (p.pair_tiles > 0) {
            // act = BF16(silu(gate) * up) of the chunk's c pair tiles
            bar_compute<NW>();
            const float* stg = reinterpret_cast<const float*>(smem + p.stg_off);
            uint16_t* act = static_cast<uint16_t*>(p.y);
            for (int i = threadIdx.x; i < c * 16 * p.batch; i += NW * 32) {
                const int bb = i / (c * 16), rr = i - bb * (c * 16);
                const int64_t row = (int64_t)r * 16 + rr;
                if (row < p.n) {
                    const float gv = stg[rr * 8 + bb], uv = stg[(c * 16 + rr) * 8 + bb];
                    act[bb * p.n + row] = float_to_bf16_bits(gv / (1.0f + expf(-gv)) * uv);
                }
            }
            bar_compute<NW>();  // the staging area is reused by the next chunk
        }
        r += c;
    }
    return true;
}

template <int FMT, int NT, int LANES, int NW, int CAP>
__global__ void __launch_bounds__(threads_of<NW>(), NW == 8 ? 2 : 1)
    gemv_rows_kernel(const __grid_constant__ Maps tm, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = ptx::align_smem<1024>(smem_raw);
    const uint32_t bar_off = p.bar_off;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + bar_off);
    uint64_t* empty = full + kMaxSlots;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = gridDim.x, c = blockIdx.x;

    if (threadIdx.x == 0) {
        for (int i = 0; i < p.slots; ++i) {
            ptx::mbar_init(&full[i], 1);
            ptx::mbar_init(&empty[i], NW);
        }
        ptx::fence_barrier_init();
    }
    __syncthreads();
    // row tiles [rt0, rt1): the first row_tiles % C CTAs take one extra
    const int tq = p.row_tiles / C, trem = p.row_tiles - tq * C;
    const int rt0 = c * tq + min(c, trem), rt1 = rt0 + tq + (c < trem ? 1 : 0);
    ptx::pdl_launch_dependents();

    if (warp == NW) {
        // ------------------------------------------------ weight producer
        // lane 0 waits for the slot and posts the byte count; the copies of a
        // stage are then issued by several lanes at once (one row tile, or one
        // 128-row box, each)
        if (lane == 0) {
            ptx::prefetch_tensormap(&tm.codes16);
            ptx::prefetch_tensormap(&tm.scales16);
            ptx::prefetch_tensormap(&tm.codes128);
            ptx::prefetch_tensormap(&tm.scales128);
        }
        int it = 0;
        Ring rp;
        rp.depth = p.slots;
        produce<FMT>(tm, p, smem, full, empty, rt0, rt1, rp, it, lane);
        // every copy this CTA issued must land before it may exit
        if (lane == 0)
            for (int j = (it > p.slots ? it - p.slots : 0); j < it; ++j)
                if (!ptx::mbar_wait_bounded(&full[j % p.slots], (uint32_t)((j / p.slots) & 1), kWaitPolls))
                    record_status(p.status, BQ_ERR_TIMEOUT);
        return;
    }

    // ---------------------------------------------------- compute warps
    if (FMT == BQ_T5P8G128) {
        // digit table: lut[32 v + l] = c0 | c1 << 8 | c2 << 16 | c3 << 24 of byte v
        uint32_t* lut = reinterpret_cast<uint32_t*>(smem + p.lut_off);
        for (int i = threadIdx.x; i < 256 * 32; i += NW * 32) {
            const uint32_t v = (uint32_t)i >> 5;
            lut[i] = (v % 3u) | ((v / 3u % 3u) << 8) | ((v / 9u % 3u) << 16) | ((v / 27u % 3u) << 24);
        }
    }
    ptx::pdl_wait();  // x is produced, y may still be read, by the previous kernel
    prep_x<FMT, NT, LANES, NW, false>(p, smem, warp, lane);
    bar_compute<NW>();
    Ring rp;
    rp.depth = p.slots;
    run_chunks<FMT, NT, LANES, NW, CAP>(p, smem, full, empty, rt0, rt1, rp, warp, lane);
}

// ------------------------------------------------------------ chain kernel
// A persistent grid (one CTA of 16 compute warps per SM) that runs a short
// list of dependent products in order -- the projections of one decoder
// layer ("1-bit Bonsai 8B" notes, Table 1: GQA attention projections and the
// SwiGLU feed-forward).  The producer warp streams every step's weights back
// to back through one ring, so the next product's weights arrive while the
// current one computes; the compute warps finish step s, publish it with a
// grid-wide barrier (a counter in global memory, bounded waits), and only then
// read step s+1's activations, which may be step s's output.  A SwiGLU step
// (W = [gate; up]) writes BF16(silu(gate) * up) instead of the raw products.
constexpr int kMaxChainSteps = 8;
constexpr int kChainStgBytes = 16 * 16 * 8 * 4;  // [16 tiles][16 rows][8 batch] floats

struct ChainMaps {
    Maps m[kMaxChainSteps];
};
struct ChainParams {
    Params step[kMaxChainSteps];  // shared-memory layout fields are the same in every step
    int nsteps;
    unsigned int* bar;            // [0] barrier arrivals, [1] exits; zero on entry, left zero
};

__device__ __forceinline__ unsigned int ld_acquire_gpu(const unsigned int* a) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
    return v;
}

// Compute warps of every CTA: publish this CTA's outputs of the current step
// (arrive), or wait until every CTA has published (target arrivals).  Only
// thread 0 touches the counter; the other threads wait at the compute-warp
// barrier.  A wait that gives up records BQ_ERR_TIMEOUT; the return value is
// the same in every compute thread.
template <int NW>
__device__ void grid_arrive(unsigned int* bar) {
    bar_compute<NW>();  // every compute thread's stores of the step are done
    if (threadIdx.x == 0) {
        // release: the CTA's stores (ordered before this thread by the barrier)
        // become visible no later than the arrival
        asm volatile("fence.acq_rel.gpu;\n\tred.relaxed.gpu.global.add.u32 [%0], 1;" ::"l"(bar) : "memory");
    }
}

template <int NW>
__device__ bool grid_wait(unsigned int* bar, unsigned int target, int* status, int* flag_smem) {
    if (threadIdx.x == 0) {
        int ok = 1;
        if (ld_acquire_gpu(&bar[0]) < target) {
            const uint64_t t0 = ptx::globaltimer_ns();
            for (uint32_t i = 1;; ++i) {
                if (i > 64) __nanosleep(32);  // poll tightly first: the release is usually close
                if (ld_acquire_gpu(&bar[0]) >= target) break;
                if (i >= kWaitPolls || ((i & 255u) == 0 && ptx::globaltimer_ns() - t0 > ptx::kWaitLimitNs)) {
                    record_status(status, BQ_ERR_TIMEOUT);
                    ok = 0;
                    break;
                }
            }
        }
        *flag_smem = ok;
    }
    bar_compute<NW>();
    return *flag_smem != 0;
}

template <int FMT, int NT, int LANES>
__global__ void __launch_bounds__(threads_of<16>(), 1)
    gemv_chain_kernel(const __grid_constant__ ChainMaps tm, const __grid_constant__ ChainParams cp) {
    constexpr int NW = 16;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = ptx::align_smem<1024>(smem_raw);
    const Params& p0 = cp.step[0];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + p0.bar_off);
    uint64_t* empty = full + kMaxSlots;
    int* flag = reinterpret_cast<int*>(smem + p0.bar_off + 2 * kMaxSlots * 8);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = gridDim.x, c = blockIdx.x;
    if (threadIdx.x == 0) {
        for (int i = 0; i < p0.slots; ++i) {
            ptx::mbar_init(&full[i], 1);
            ptx::mbar_init(&empty[i], NW);
        }
        ptx::fence_barrier_init();
    }
    __syncthreads();
    // (every CTA of this grid is resident once all of them have executed
    // this, so a later kernel cannot take an SM one of them still needs)
    ptx::pdl_launch_dependents();
    const int nsteps = cp.nsteps;

    if (warp == NW) {
        // ------------------------------------------------ weight producer
        if (lane < 4 * nsteps) {
            const Maps& m = tm.m[lane >> 2];
            const CUtensorMap* mp[4] = {&m.codes16, &m.scales16, &m.codes128, &m.scales128};
            ptx::prefetch_tensormap(mp[lane & 3]);
        }
        int it = 0;
        Ring rp;
        rp.depth = p0.slots;
        for (int s = 0; s < nsteps; ++s) {
            const Params& p = cp.step[s];
            const int tq = p.row_tiles / C, trem = p.row_tiles - tq * C;
            const int rt0 = c * tq + min(c, trem), rt1 = rt0 + tq + (c < trem ? 1 : 0);
            if (!produce<FMT>(tm.m[s], p, smem, full, empty, rt0, rt1, rp, it, lane)) break;
        }
        if (lane == 0)
            for (int j = (it > p0.slots ? it - p0.slots : 0); j < it; ++j)
                if (!ptx::mbar_wait_bounded(&full[j % p0.slots], (uint32_t)((j / p0.slots) & 1), kWaitPolls))
                    record_status(p0.status, BQ_ERR_TIMEOUT);
        return;
    }

    // ---------------------------------------------------- compute warps
    if (FMT == BQ_T5P8G128) {
        uint32_t* lut = reinterpret_cast<uint32_t*>(smem + p0.lut_off);
        for (int i = threadIdx.x; i < 256 * 32; i += NW * 32) {
            const uint32_t v = (uint32_t)i >> 5;
            lut[i] = (v % 3u) | ((v / 3u % 3u) << 8) | ((v / 9u % 3u) << 16) | ((v / 27u % 3u) << 24);
        }
    }
    ptx::pdl_wait();  // the first step's x is produced, the outputs may still be read, by the previous kernel
    Ring rp;
    rp.depth = p0.slots;
    bool ok = true;
    for (int s = 0; s < nsteps && ok; ++s) {
        const Params& p = cp.step[s];
        if (s > 0) ok = grid_wait<NW>(cp.bar, (unsigned int)(s * C), p0.status, flag);
        if (!ok) break;
        prep_x<FMT, NT, LANES, NW, true>(p, smem, warp, lane);
        bar_compute<NW>();
        const int tq = p.row_tiles / C, trem = p.row_tiles - tq * C;
        const int rt0 = c * tq + min(c, trem), rt1 = rt0 + tq + (c < trem ? 1 : 0);
        ok = run_chunks<FMT, NT, LANES, NW>(p, smem, full, empty, rt0, rt1, rp, warp, lane);
        if (s + 1 < nsteps) grid_arrive<NW>(cp.bar);
    }
    // The last CTA out leaves the counters zero for the next launch (every CTA
    // has passed its last wait by then).
    bar_compute<NW>();
    if (threadIdx.x == 0 && ok) {
        __threadfence();
        if (atomicAdd(&cp.bar[1], 1u) == (unsigned int)C - 1) {
            atomicExch(&cp.bar[0], 0u);
            atomicExch(&cp.bar[1], 0u);
        }
    }
}

// ------------------------------------------------------- wide-batch decode
// Batch 5..16, binary and 2-bit ternary (and 5-trit, whose codes become the
// same FP16 pairs through base-3 quotient arithmetic).  The weights become exact FP16
// effective weights s * q inside the A registers of the warp MMA m16n8k16:
//   binary: ((w << (15 - m)) & 0x80008000) ^ (s | s << 16) ^ 0x80008000 is the
//           pair (weight m, weight m + 16) of code word w as (+-s, +-s), the
//           sign the negated bit (bit 1 -> +s);
//   2-bit : the codes c of weights i and i + 8 of a word placed in the low bits
//           of the FP16 1024 give 1024 + c; minus 1025 is q = c - 1, times s is
//           s * q, all exact;
// and x enters as FP16 x * 2^e_b with one power of two per batch row b (its
// largest |x| in [2^14, 2^15): exact for every BF16 value within 2^-31 of the
// row's largest magnitude), so the MMA accumulates s * q * x over all of K in
// FP32 and y = acc * 2^-e_b -- no per-group recombination and no digit split:
// one decoded 16 x 16 weight fragment feeds one MMA per 8 batch rows.
constexpr int kWideAux = 256;  // per batch row: largest |x|, 2^e as two factors, 2^-e

// Activation area per stage: [group G][j 0..7][batch row b][thread t][2 words],
// word p of (G, b, t) the FP16 pair of the two activations register p of a
// weight row pairs (see wide_lo / wide_hi); MMA j reads words 2j, 2j + 1.
template <int NTW>
__host__ __device__ constexpr int wide_stage_bytes() { return kGroupsPerStage * 8 * (NTW * 8) * 4 * 8; }

// The weights of register p (0..15) of a thread's weight row, as indices r
// into the thread's 32 weights of the group: binary (p, p + 16) and 2-bit
// p < 8: (p, p + 8), else (p + 8, p + 16), with weight r at k = 32 t + r;
// 5-trit p < 15: (p, p + 15), digit p % 5 of bytes 6 t + p / 5 and
// 6 t + p / 5 + 3, and p = 15: (30, 31), the thread's two trits of the group's
// last eight (weight r < 30 at k = 30 t + r, r = 30, 31 at k = 120 + 2 t + r - 30;
// the row-owning kernel's split of the 26 bytes).
template <int FMT>
__device__ __forceinline__ constexpr int wide_lo(int p) {
    return FMT == BQ_T2G128 ? (p < 8 ? p : p + 8) : FMT == BQ_T5P8G128 ? (p < 15 ? p : 30) : p;
}
template <int FMT>
__device__ __forceinline__ constexpr int wide_hi(int p) {
    return FMT == BQ_T2G128 ? (p < 8 ? p + 8 : p + 16) : FMT == BQ_T5P8G128 ? (p < 15 ? p + 15 : 31) : p + 16;
}

// x -> the FP16 activation area of all of K, per-row power-of-two pre-scale.
template <int FMT, int NTW, int NW>
__device__ __forceinline__ void prep_wide(const Params& p, uint8_t* smem) {
    constexpr int BP = NTW * 8;
    const int tid = threadIdx.x;
    uint32_t* rmax = reinterpret_cast<uint32_t*>(smem + p.lut_off);
    float2* fac = reinterpret_cast<float2*>(smem + p.lut_off + 64);  // 2^e as two exact factors
    float* inv = reinterpret_cast<float*>(smem + p.lut_off + 192);
    if (tid < BP) rmax[tid] = 0u;
    bar_compute<NW>();
    // largest |x| of every batch row (FP32 bits of the magnitude: monotonic):
    // one warp per row, its loads unrolled so that they are in flight together
    // (a loop over the rows with all threads on one row waited one L2 round
    // trip per row)
    const int64_t c8 = p.k / 8;
    for (int b = tid >> 5; b < p.batch; b += NW) {
        uint32_t m = 0u;
        const uint4* row = reinterpret_cast<const uint4*>(p.x + b * p.k);
#pragma unroll 16
        for (int64_t c = tid & 31; c < c8; c += 32) {
            const uint4 v = __ldg(row + c);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) m = max(m, max((w[q] << 16) & 0x7FFFFFFFu, w[q] & 0x7FFF0000u));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
        if ((tid & 31) == 0) rmax[b] = m;
    }
    bar_compute<NW>();
    if (tid < BP) {
        const float m = __uint_as_float(rmax[tid]);
        const int e = m > 0.f ? 14 - ilog2f(m) : 0;  // in [-113, 147]
        const int e1 = min(e, 127);                   // 2^e = 2^e1 2^(e - e1), both normal
        fac[tid] = make_float2(__int_as_float((e1 + 127) << 23), __int_as_float((e - e1 + 127) << 23));
        inv[tid] = ldexpf(1.0f, -e);  // exact (a subnormal below 2^-126)
    }
    bar_compute<NW>();
    // (stage, group, batch row, thread t): 32 activations -> 16 FP16 pairs
    uint8_t* xres = smem + p.x_off;
    const int tasks = p.stages * kGroupsPerStage * BP * 4;
#pragma unroll 2
    for (int i = tid; i < tasks; i += NW * 32) {
        const int t = i & 3, b = (i >> 2) % BP, rest = i / (4 * BP), G = rest & 7, st = rest >> 3;
        uint32_t words[16];
        if (b < p.batch) {
            uint32_t raw[16];
            if (FMT == BQ_T5P8G128) {
                // weights 30 t .. 30 t + 29 and 120 + 2 t, 121 + 2 t (4-byte aligned)
                const uint16_t* xg = p.x + b * p.k + st * 1024 + G * 128;
                const uint32_t* src = reinterpret_cast<const uint32_t*>(xg + 30 * t);
#pragma unroll
                for (int q = 0; q < 15; ++q) raw[q] = __ldg(src + q);
                raw[15] = __ldg(reinterpret_cast<const uint32_t*>(xg + 120 + 2 * t));
            } else {
                const uint4* src = reinterpret_cast<const uint4*>(p.x + b * p.k + st * 1024 + G * 128 + 32 * t);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4 v = __ldg(src + q);
                    raw[4 * q] = v.x; raw[4 * q + 1] = v.y; raw[4 * q + 2] = v.z; raw[4 * q + 3] = v.w;
                }
            }
            // x 2^e rounded once to FP16 (the two power-of-two products are
            // exact while the value stays in the FP32 normal range; below it
            // the FP16 result is zero either way)
            const float2 f = fac[b];
            float v[32];
#pragma unroll
            for (int r = 0; r < 32; ++r)
                v[r] = __uint_as_float((r & 1) ? (raw[r >> 1] & 0xFFFF0000u) : (raw[r >> 1] << 16)) * f.x * f.y;
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                uint32_t w2;
                asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(w2) : "f"(v[wide_hi<FMT>(q)]), "f"(v[wide_lo<FMT>(q)]));
                words[q] = w2;
            }
        } else {
#pragma unroll
            for (int q = 0; q < 16; ++q) words[q] = 0u;
        }
        uint8_t* base = xres + (size_t)st * wide_stage_bytes<NTW>();
#pragma unroll
        for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint2*>(base + ((((G * 8 + j) * BP + b) * 4 + t) * 8)) =
                make_uint2(words[2 * j], words[2 * j + 1]);
    }
}

__device__ __forceinline__ __half2 u2h2(uint32_t u) {
    __half2 h;
    *reinterpret_cast<uint32_t*>(&h) = u;
    return h;
}
__device__ __forceinline__ uint32_t h22u(__half2 h) { return *reinterpret_cast<const uint32_t*>(&h); }

// The four A registers of MMA j for rows g (w: its code words) and g + 8
// (wb), scales S (binary: (s | s << 16) ^ 0x80008000; 2-bit: s | s << 16).
template <int FMT>
__device__ __forceinline__ void wide_a(uint2 w, uint2 wb, uint32_t S, uint32_t Sb, int j, uint32_t (&a)[4]) {
    if (FMT == BQ_Q1G128) {
        const int m0 = 2 * j, m1 = 2 * j + 1;
        a[0] = ((w.x << (15 - m0)) & 0x80008000u) ^ S;
        a[1] = ((wb.x << (15 - m0)) & 0x80008000u) ^ Sb;
        a[2] = ((w.x << (15 - m1)) & 0x80008000u) ^ S;
        a[3] = ((wb.x << (15 - m1)) & 0x80008000u) ^ Sb;
    } else {
        const __half2 k1025 = u2h2(0x64016401u);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int pr = 2 * j + h;  // register pair p
            const uint32_t word = pr < 8 ? w.x : w.y, wordb = pr < 8 ? wb.x : wb.y;
            const int sh = 2 * (pr & 7);
            const __half2 qa = __hsub2(u2h2(((word >> sh) & 0x00030003u) | 0x64006400u), k1025);
            const __half2 qb = __hsub2(u2h2(((wordb >> sh) & 0x00030003u) | 0x64006400u), k1025);
            a[2 * h] = h22u(__hmul2(qa, u2h2(S)));
            a[2 * h + 1] = h22u(__hmul2(qb, u2h2(Sb)));
        }
    }
}

// 5-trit format: (c - 1) s of two codes c in {0, 1, 2} held in the halves of
// c2, as an FP16 pair: (1024 + c) - 1025 = c - 1 exactly, times s exactly.
__device__ __forceinline__ uint32_t t5_qpair(uint32_t c2, uint32_t S) {
    const __half2 q = __hsub2(u2h2(c2 | 0x64006400u), u2h2(0x64016401u));
    return h22u(__hmul2(q, u2h2(S)));
}

// The five base-3 digits of the two bytes in the halves of v: quotients
// floor(v / 3^i) by multiply-shift (171 >> 9, 57 >> 9, 19 >> 9, 203 >> 14, exact
// for every byte; v * m < 2^16, so the halves do not mix once masked), digit i
// = q_i - 3 q_(i+1) (never negative, so no borrow between the halves).
__device__ __forceinline__ void t5_digits5(uint32_t v, uint32_t (&d)[5]) {
    const uint32_t q1 = ((v * 171u) >> 9) & 0x007F007Fu, q2 = ((v * 57u) >> 9) & 0x007F007Fu;
    const uint32_t q3 = ((v * 19u) >> 9) & 0x007F007Fu, q4 = ((v * 203u) >> 14) & 0x00030003u;
    d[0] = v - 3u * q1;
    d[1] = q1 - 3u * q2;
    d[2] = q2 - 3u * q3;
    d[3] = q3 - 3u * q4;
    d[4] = q4;
}

// The 16 FP16 pairs of one row's group for thread t (pairs as wide_lo /
// wide_hi): bytes 6t .. 6t+5 paired (j, j + 3) in 16-bit halves, and the
// thread's two trits of the last eight (bytes 24, 25).  p: the group's 26
// bytes in shared memory (2-byte aligned); S: the row's FP16 scale in both
// halves.
__device__ __forceinline__ void t5_wide_row(const uint8_t* p, int t, uint32_t S, uint32_t (&h)[16]) {
    const uint32_t u0 = lds_u16(p + 6 * t), u1 = lds_u16(p + 6 * t + 2), u2 = lds_u16(p + 6 * t + 4);
    const uint32_t ue = lds_u16(p + 24);
    const uint32_t xs[3] = {(u0 & 0xFFu) | ((u1 >> 8) << 16), (u0 >> 8) | ((u2 & 0xFFu) << 16),
                            (u1 & 0xFFu) | ((u2 >> 8) << 16)};
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        uint32_t d[5];
        t5_digits5(xs[j], d);
#pragma unroll
        for (int i = 0; i < 5; ++i) h[5 * j + i] = t5_qpair(d[i], S);
    }
    // byte 24 (trits 120..124) in the low half, byte 25 (125..127) in the high
    uint32_t e[5];
    t5_digits5((ue & 0xFFu) | ((ue >> 8) << 16), e);
    const uint32_t c0 = (e[0] & 0xFFFFu) | (e[1] << 16), c1 = (e[2] & 0xFFFFu) | (e[3] << 16);
    const uint32_t c2 = (e[4] & 0xFFFFu) | (e[0] & 0xFFFF0000u), c3 = (e[1] >> 16) | (e[2] & 0xFFFF0000u);
    h[15] = t5_qpair(t == 0 ? c0 : t == 1 ? c1 : t == 2 ? c2 : c3, S);
}

// One chunk of CT row tiles, all stages, accumulating in FP32 across K; work
// split as run_chunk.
template <int FMT, int NTW, int NW, int CT>
__device__ bool run_chunk_wide(const Params& p, uint8_t* smem, uint64_t* full, uint64_t* empty, int rt, Ring& rp,
                               int warp, int lane, int ct) {
    constexpr int TPW = CT >= NW ? CT / NW : 1;
    constexpr int WPR = CT >= NW ? 1 : ((NW / CT) < kGroupsPerStage ? (NW / CT) : kGroupsPerStage);
    constexpr int GPW = kGroupsPerStage / WPR;
    constexpr int BP = NTW * 8;
    // code bytes between row tiles (of a column box for the bit formats)
    constexpr int TSTRIDE = FMT == BQ_T5P8G128 ? tile_code_bytes<FMT>() : 2048;
    const int my_rt = CT >= NW ? warp : warp / WPR;
    const int gsub = CT >= NW ? 0 : warp % WPR;
    const bool active = my_rt < ct;  // (ct <= CT tiles in the chunk; as in run_chunk)
    const int g = lane >> 2, t = lane & 3;
    float acc[TPW][NTW][4];
#pragma unroll
    for (int tp = 0; tp < TPW; ++tp)
#pragma unroll
        for (int nt = 0; nt < NTW; ++nt)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[tp][nt][c] = 0.0f;
    bool alive = true;
    for (int st = 0; st < p.stages; ++st) {
        const int slot = rp.slot;
        if (!ptx::mbar_wait_bounded(&full[slot], rp.round & 1u, kWaitPolls)) {
            record_status(p.status, BQ_ERR_TIMEOUT);
            alive = false;
            break;
        }
        rp.next();
        if (active) {
            const uint8_t* sb = smem + slot * p.slot_bytes;
            const uint8_t* xs = smem + p.x_off + (size_t)st * wide_stage_bytes<NTW>();
            uint32_t sc[TPW][2][(GPW + 1) / 2];
#pragma unroll
            for (int tp = 0; tp < TPW; ++tp) {
                const uint8_t* srow = sb + p.scales_off + (my_rt + NW * tp) * kTileScaleBytes + gsub * GPW * 2;
                load_scales<GPW>(srow + g * 16, sc[tp][0]);
                load_scales<GPW>(srow + (g + 8) * 16, sc[tp][1]);
            }
#pragma unroll
            for (int gi = 0; gi < GPW; ++gi) {
                const int G = gsub * GPW + gi;
#pragma unroll
                for (int tp = 0; tp < TPW; ++tp) {
                    const uint8_t* codes_t = sb + (my_rt + NW * tp) * TSTRIDE;
                    if constexpr (FMT == BQ_T5P8G128) {
                        const uint32_t s0 = (sc[tp][0][gi >> 1] >> (16 * (gi & 1))) & 0xFFFFu;
                        const uint32_t s1 = (sc[tp][1][gi >> 1] >> (16 * (gi & 1))) & 0xFFFFu;
                        const uint8_t* r0 = codes_t + g * kT5RowBytes + 26 * G;
                        uint32_t h0[16], h1[16];
                        t5_wide_row(r0, t, s0 | (s0 << 16), h0);
                        t5_wide_row(r0 + 8 * kT5RowBytes, t, s1 | (s1 << 16), h1);
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
#pragma unroll
                            for (int nt = 0; nt < NTW; ++nt) {
                                const uint2 bv = *reinterpret_cast<const uint2*>(
                                    xs + ((((G * 8 + j) * BP + nt * 8 + g) * 4 + t) * 8));
                                ptx::mma_f16_16816(acc[tp][nt], h0[2 * j], h1[2 * j], h0[2 * j + 1], h1[2 * j + 1],
                                                   bv.x, bv.y);
                            }
                        }
                        continue;
                    }
                    uint2 w, wb;
                    if (FMT == BQ_Q1G128) {
                        const int off = ((G ^ g) << 4) + 4 * t;
                        w = make_uint2(*reinterpret_cast<const uint32_t*>(codes_t + g * 128 + off), 0u);
                        wb = make_uint2(*reinterpret_cast<const uint32_t*>(codes_t + (g + 8) * 128 + off), 0u);
                    } else {
                        const uint8_t* box = codes_t + (G >> 2) * (p.chunk_cap * 2048);
                        const int chunk = 2 * (G & 3) + (t >> 1);
                        const int off = ((chunk ^ g) << 4) + 8 * (t & 1);
                        w = *reinterpret_cast<const uint2*>(box + g * 128 + off);
                        wb = *reinterpret_cast<const uint2*>(box + (g + 8) * 128 + off);
                    }
                    const uint32_t s0 = (sc[tp][0][gi >> 1] >> (16 * (gi & 1))) & 0xFFFFu;
                    const uint32_t s1 = (sc[tp][1][gi >> 1] >> (16 * (gi & 1))) & 0xFFFFu;
                    const uint32_t flip = FMT == BQ_Q1G128 ? 0x80008000u : 0u;
                    const uint32_t S = (s0 | (s0 << 16)) ^ flip, Sb = (s1 | (s1 << 16)) ^ flip;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        uint32_t a[4];
                        wide_a<FMT>(w, wb, S, Sb, j, a);
#pragma unroll
                        for (int nt = 0; nt < NTW; ++nt) {
                            const uint2 bv = *reinterpret_cast<const uint2*>(
                                xs + ((((G * 8 + j) * BP + nt * 8 + g) * 4 + t) * 8));
                            ptx::mma_f16_16816(acc[tp][nt], a[0], a[1], a[2], a[3], bv.x, bv.y);
                        }
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&empty[slot]);
    }
    if (WPR > 1) {
        float* red = reinterpret_cast<float*>(smem + p.red_off);
#pragma unroll
        for (int nt = 0; nt < NTW; ++nt)
#pragma unroll
            for (int c = 0; c < 4; ++c) red[((warp * 32 + lane) * NTW + nt) * 4 + c] = acc[0][nt][c];
        bar_compute<NW>();
        if (active && gsub == 0) {
#pragma unroll
            for (int nt = 0; nt < NTW; ++nt)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float sum = 0.0f;
#pragma unroll
                    for (int q = 0; q < WPR; ++q) sum += red[(((warp + q) * 32 + lane) * NTW + nt) * 4 + c];
                    acc[0][nt][c] = sum;
                }
        }
        bar_compute<NW>();
    }
    if (active && gsub == 0) {
        const float* inv = reinterpret_cast<const float*>(smem + p.lut_off + 192);
#pragma unroll
        for (int tp = 0; tp < TPW; ++tp)
#pragma unroll
            for (int nt = 0; nt < NTW; ++nt)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int bb = nt * 8 + 2 * t + (c & 1);
                    const int64_t row = (int64_t)(rt + my_rt + NW * tp) * 16 + g + 8 * (c >> 1);
                    if (bb < p.batch && row < p.n && my_rt + NW * tp < ct) {
                        const float v = acc[tp][nt][c] * inv[bb];
                        if (p.y_dtype == BQ_F32)
                            static_cast<float*>(p.y)[bb * p.n + row] = v;
                        else
                            static_cast<uint16_t*>(p.y)[bb * p.n + row] = float_to_bf16_bits(v);
                    }
                }
    }
    return alive;
}

template <int FMT, int NTW, int CAP>
__global__ void __launch_bounds__(threads_of<16>(), 1)
    gemv_wide_kernel(const __grid_constant__ Maps tm, const Params p) {
    constexpr int NW = 16;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = ptx::align_smem<1024>(smem_raw);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.bar_off);
    uint64_t* empty = full + kMaxSlots;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = gridDim.x, c = blockIdx.x;
    if (threadIdx.x == 0) {
        for (int i = 0; i < p.slots; ++i) {
            ptx::mbar_init(&full[i], 1);
            ptx::mbar_init(&empty[i], NW);
        }
        ptx::fence_barrier_init();
    }
    __syncthreads();
    const int tq = p.row_tiles / C, trem = p.row_tiles - tq * C;
    const int rt0 = c * tq + min(c, trem), rt1 = rt0 + tq + (c < trem ? 1 : 0);
    ptx::pdl_launch_dependents();
    if (warp == NW) {
        if (lane == 0) {
            ptx::prefetch_tensormap(&tm.codes16);
            ptx::prefetch_tensormap(&tm.scales16);
            ptx::prefetch_tensormap(&tm.codes128);
            ptx::prefetch_tensormap(&tm.scales128);
        }
        int it = 0;
        Ring rp;
        rp.depth = p.slots;
        produce<FMT>(tm, p, smem, full, empty, rt0, rt1, rp, it, lane);
        if (lane == 0)
            for (int j = (it > p.slots ? it - p.slots : 0); j < it; ++j)
                if (!ptx::mbar_wait_bounded(&full[j % p.slots], (uint32_t)((j / p.slots) & 1), kWaitPolls))
                    record_status(p.status, BQ_ERR_TIMEOUT);
        return;
    }
    ptx::pdl_wait();  // x is produced, y may still be read, by the previous kernel
    prep_wide<FMT, NTW, NW>(p, smem);
    bar_compute<NW>();
    Ring rp;
    rp.depth = p.slots;
    for (int r = rt0; r < rt1;) {
        // any tile count, in the compiled shape of the next power of two
        const int ct = chunk_count(rt1 - r, p.chunk_cap);
        bool ok;
        if (CAP >= 8 && ct > 4)
            ok = run_chunk_wide<FMT, NTW, NW, CAP >= 8 ? 8 : 1>(p, smem, full, empty, r, rp, warp, lane, ct);
        else if (CAP >= 4 && ct > 2)
            ok = run_chunk_wide<FMT, NTW, NW, CAP >= 4 ? 4 : 1>(p, smem, full, empty, r, rp, warp, lane, ct);
        else if (ct == 2)
            ok = run_chunk_wide<FMT, NTW, NW, 2>(p, smem, full, empty, r, rp, warp, lane, ct);
        else
            ok = run_chunk_wide<FMT, NTW, NW, 1>(p, smem, full, empty, r, rp, warp, lane, ct);
        if (!ok) break;
        r += ct;
    }
}

// ----------------------------------------------------------------- host
struct Plan {
    int nt = 0, lanes = 0, nw = 0, stages = 0, row_tiles = 0, slots = 0, grid = 0, chunk_cap = 8, slot_bytes = 0,
        scales_off = 0;
    uint32_t x_off = 0, red_off = 0, lut_off = 0, bar_off = 0, smem = 0;
    bool ok = false;
};

// Shared-memory layout for NW compute warps within `limit` bytes; false if a
// ring of two slots does not fit.
bool layout(Plan& pl, int fmt, int nw, int limit, int sms) {
    const int ctas_per_sm = nw == 8 ? 2 : 1;
    const int cap_grid = sms * ctas_per_sm;
    pl.nw = nw;
    pl.grid = pl.row_tiles < cap_grid ? pl.row_tiles : cap_grid;
    // 16-tile chunks (binary, batch <= 4) where a CTA owns more than 8 row
    // tiles (9..15 tiles run as one 16-tile chunk: measured faster than 8 plus
    // the rest); otherwise 8-tile slots keep the ring deep.  A chunk is the
    // smallest power of two that holds the most tiles a CTA owns (e.g. 3 tiles
    // run as one 4-tile chunk with one tile idle), or, where that leaves the
    // ring fewer than two slots, the largest power of two within those tiles; a
    // slot is a multiple of 1 KB (the swizzled copies land on 1 KB boundaries).
    const int64_t tsb = kTileScaleBytes * (fmt == BQ_A1G128 ? 2 : 1);
    const bool bits = fmt == BQ_Q1G128 || fmt == BQ_A1G128;
    const int64_t tile_bytes = (bits ? 2048 : fmt == BQ_T2G128 ? 4096 : 16 * kT5RowBytes) + tsb;
    const int top = (bits && pl.nt <= 2 && pl.row_tiles / pl.grid >= 9) ? 16 : kMaxChunkTiles;
    const int most = (pl.row_tiles + pl.grid - 1) / pl.grid;
    int within = top;  // largest power of two <= most
    while (within > 1 && within > most) within >>= 1;
    pl.chunk_cap = top;  // smallest power of two >= most
    while (pl.chunk_cap > 1 && pl.chunk_cap / 2 >= most) pl.chunk_cap >>= 1;
    const int64_t lut = fmt == BQ_T5P8G128 ? kLutBytes : 0;
    const int64_t x_area = ((int64_t)pl.stages * pl.nt * x_nt_bytes(pl.lanes) + 1023) / 1024 * 1024;
    const int64_t red = (int64_t)nw * 32 * pl.nt * 2 * 4;
    const int64_t fixed = 1024 + x_area + red + lut + 2 * kMaxSlots * 8;
    int64_t slot = 0, slots = 0;
    for (;;) {
        slot = (pl.chunk_cap * tile_bytes + 1023) / 1024 * 1024;
        slots = (limit - fixed) / slot;
        if (slots >= 2 || pl.chunk_cap == within) break;
        pl.chunk_cap = within;
    }
    pl.slot_bytes = (int)slot;
    pl.scales_off = pl.chunk_cap * (int)(tile_bytes - tsb);
    if (slots > kMaxSlots) slots = kMaxSlots;
    if (slots < 2) return false;
    pl.slots = (int)slots;
    pl.x_off = (uint32_t)(slots * slot);
    pl.red_off = (uint32_t)(pl.x_off + x_area);
    pl.lut_off = (uint32_t)(pl.red_off + red);
    pl.bar_off = (uint32_t)(pl.lut_off + lut);
    pl.smem = (uint32_t)(1024 + pl.bar_off + 2 * kMaxSlots * 8);
    return true;
}

Plan make_plan(int fmt, int64_t n, int64_t k, int batch) {
    Plan pl;
    if (!((fmt == BQ_Q1G128 || fmt == BQ_T2G128 || fmt == BQ_T5P8G128 || fmt == BQ_A1G128) && batch >= 1 &&
          batch <= 8 && k > 0 &&
          k % 1024 == 0 && n > 0 &&
          n <= (int64_t)INT32_MAX - 16 && k / 4 <= (int64_t)INT32_MAX / 4 && k <= (int64_t)1 << 20))
        return pl;
    pl.nt = batch <= 2 ? 1 : batch <= 4 ? 2 : 4;  // n-tiles of two batch rows (5..8 -> 4)
    pl.lanes = batch == 1 ? 16 : 32;
    pl.stages = (int)(k / 1024);
    pl.row_tiles = (int)((n + 15) / 16);
    const int sms = sm_count();
    // Two CTAs per SM (8 compute warps, half the shared memory each) for the
    // largest matrices (at least 32 row tiles per SM), where the activation
    // operand leaves room for a ring; else one CTA of 16 compute warps per SM.
    // (Measured on B200: the half-SM shape on every call let each call's CTAs
    // prefetch under the previous call, but the 8-warp compute of the small
    // and medium matrices lost more than that gained; on the largest matrices
    // two 8-warp CTAs per SM, each with two row tiles per warp, are faster.)
    if (pl.nt == 1 && pl.row_tiles >= 32 * sms && layout(pl, fmt, 8, kSmemHalf, sms)) {
        pl.ok = true;
        return pl;
    }
    pl.ok = layout(pl, fmt, 16, kSmemFull, sms);
    return pl;
}

template <int FMT, int NT, int LANES, int NW, int CAP>
cudaError_t launch_typed(const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k, const uint16_t* x,
                         int batch, void* y, int y_dtype, const Plan& pl, cudaStream_t s) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    {
        const cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(gemv_rows_kernel<FMT, NT, LANES, NW, CAP>),
                                                  NW == 8 ? kSmemHalf : kSmemFull);
        if (e != cudaSuccess) return e;
    }
    const int64_t row_bytes = bits_fmt<FMT>() ? k / 8 : (FMT == BQ_T2G128) ? k / 4 : (k / 128) * 26;
    const int64_t G = k / 128;
    Maps tm;
    for (int v = 0; v < 2; ++v) {
        const cuuint32_t rows = v == 0 ? 16u : 128u;
        {
            cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)n};
            cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
            // 5-trit rows: 208-byte boxes, unswizzled (the 128-byte swizzle needs <= 128-byte boxes)
            cuuint32_t box[2] = {FMT == BQ_T5P8G128 ? (cuuint32_t)kT5RowBytes : 128u, rows};
            cuuint32_t es[2] = {1, 1};
            if (enc(v == 0 ? &tm.codes16 : &tm.codes128, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes),
                    dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    FMT == BQ_T5P8G128 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
        }
        {
            // the scale plane: [N][G] FP16, or [N][G][2] (scale, bias) pairs
            cuuint64_t dims[2] = {(cuuint64_t)(G * spg<FMT>()), (cuuint64_t)n};
            cuuint64_t strides[1] = {(cuuint64_t)(G * 2 * spg<FMT>())};
            cuuint32_t box[2] = {(cuuint32_t)(kGroupsPerStage * spg<FMT>()), rows};
            cuuint32_t es[2] = {1, 1};
            if (enc(v == 0 ? &tm.scales16 : &tm.scales128, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2,
                    const_cast<uint16_t*>(scales), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
        }
    }
    Params prm;
    prm.x = x;
    prm.y = y;
    prm.n = n;
    prm.k = k;
    prm.batch = batch;
    prm.y_dtype = y_dtype;
    prm.stages = pl.stages;
    prm.row_tiles = pl.row_tiles;
    prm.slots = pl.slots;
    prm.slot_bytes = pl.slot_bytes;
    prm.scales_off = pl.scales_off;
    prm.chunk_cap = pl.chunk_cap;
    prm.x_off = pl.x_off;
    prm.red_off = pl.red_off;
    prm.lut_off = pl.lut_off;
    prm.bar_off = pl.bar_off;
    prm.pair_tiles = 0;
    prm.stg_off = 0;
    prm.status = device_status_ptr();
    if (!prm.status) return cudaErrorUnknown;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.grid);
    cfg.blockDim = dim3(threads_of<NW>());
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = s;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, gemv_rows_kernel<FMT, NT, LANES, NW, CAP>, tm, prm);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int FMT, int CAP>
cudaError_t launch_cap(const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k, const uint16_t* x,
                       int batch, void* y, int y_dtype, const Plan& pl, cudaStream_t s) {
    if (pl.nw == 8) {
        if (batch == 1) return launch_typed<FMT, 1, 16, 8, CAP>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
        return launch_typed<FMT, 1, 32, 8, CAP>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
    }
    if (batch == 1) return launch_typed<FMT, 1, 16, 16, CAP>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
    if (pl.nt == 1) return launch_typed<FMT, 1, 32, 16, CAP>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
    if (pl.nt == 2) return launch_typed<FMT, 2, 32, 16, CAP>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
    return launch_typed<FMT, 4, 32, 16, CAP>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
}

// The kernel is built per largest chunk: 2 (chunks of 2 and 1 tiles), 4 (4, 2,
// 1), 8 (8, 4, 2, 1) or 16 (every chunk shape).
template <int FMT>
cudaError_t launch_fmt(const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k, const uint16_t* x,
                       int batch, void* y, int y_dtype, const Plan& pl, cudaStream_t s) {
    if (pl.chunk_cap <= 2) return launch_cap<FMT, 2>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
    if (pl.chunk_cap <= 4) return launch_cap<FMT, 4>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
    if (pl.chunk_cap <= 8) return launch_cap<FMT, 8>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
    return launch_cap<FMT, 16>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
}

}  // namespace rows

bool gemv_rows_eligible(int fmt, int64_t n, int64_t k, int batch) { return rows::make_plan(fmt, n, k, batch).ok; }

namespace rows {

cudaError_t encode_maps(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k, Maps& tm);

// Wide-batch plan: one CTA of 16 compute warps per SM, the FP16 activation
// area of all of K resident, a ring of at least two 8-tile slots.
bool wide_plan(Plan& pl, int fmt, int64_t n, int64_t k, int batch) {
    if (!((fmt == BQ_Q1G128 || fmt == BQ_T2G128 || fmt == BQ_T5P8G128) && batch >= 5 && batch <= 16 && k > 0 &&
          k % 1024 == 0 &&
          n > 0 && n <= (int64_t)INT32_MAX - 16 && k <= (int64_t)1 << 20))
        return false;
    pl.nt = batch <= 8 ? 1 : 2;  // n-tiles of eight batch rows
    pl.lanes = 0;
    pl.nw = 16;
    pl.stages = (int)(k / 1024);
    pl.row_tiles = (int)((n + 15) / 16);
    const int sms = sm_count();
    pl.grid = pl.row_tiles < sms ? pl.row_tiles : sms;
    const int64_t tile_bytes = (fmt == BQ_Q1G128 ? 2048 : fmt == BQ_T2G128 ? 4096 : 16 * kT5RowBytes) + kTileScaleBytes;
    // chunks as in the row-owning kernel: the smallest power of two that holds
    // a CTA's tiles, else (ring of fewer than two slots) the largest within them
    const int most = (pl.row_tiles + pl.grid - 1) / pl.grid;
    int within = kMaxChunkTiles;
    while (within > 1 && within > most) within >>= 1;
    pl.chunk_cap = kMaxChunkTiles;
    while (pl.chunk_cap > 1 && pl.chunk_cap / 2 >= most) pl.chunk_cap >>= 1;
    const int64_t x_area = (int64_t)pl.stages * (pl.nt == 1 ? wide_stage_bytes<1>() : wide_stage_bytes<2>());
    const int64_t red = (int64_t)16 * 32 * pl.nt * 4 * 4;
    const int64_t fixed = 1024 + x_area + red + kWideAux + 2 * kMaxSlots * 8;
    // (and below that, halved while the activations leave room for fewer than
    // two slots: a shallow ring of small chunks, e.g. 5-trit codes at K = 5120
    // and batch 16, rather than the GEMM)
    int64_t slot = (pl.chunk_cap * tile_bytes + 1023) / 1024 * 1024;
    if ((kSmemFull - fixed) / slot < 2 && pl.chunk_cap != within) pl.chunk_cap = within;
    for (;;) {
        slot = (pl.chunk_cap * tile_bytes + 1023) / 1024 * 1024;
        if ((kSmemFull - fixed) / slot >= 2 || pl.chunk_cap == 1) break;
        pl.chunk_cap >>= 1;
    }
    pl.slot_bytes = (int)slot;
    pl.scales_off = pl.chunk_cap * (int)(tile_bytes - kTileScaleBytes);
    int64_t slots = (kSmemFull - fixed) / slot;
    if (slots > kMaxSlots) slots = kMaxSlots;
    if (slots < 2) return false;
    pl.slots = (int)slots;
    pl.x_off = (uint32_t)(slots * slot);
    pl.red_off = (uint32_t)(pl.x_off + x_area);
    pl.lut_off = (uint32_t)(pl.red_off + red);  // the per-row pre-scale area
    pl.bar_off = (uint32_t)(pl.lut_off + kWideAux);
    pl.smem = (uint32_t)(1024 + pl.bar_off + 2 * kMaxSlots * 8);
    pl.ok = true;
    return true;
}

template <int FMT, int NTW, int CAP>
cudaError_t launch_wide_typed(const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k, const uint16_t* x,
                              int batch, void* y, int y_dtype, const Plan& pl, cudaStream_t s) {
    {
        const cudaError_t e =
            ensure_dynamic_smem(reinterpret_cast<const void*>(gemv_wide_kernel<FMT, NTW, CAP>), kSmemFull);
        if (e != cudaSuccess) return e;
    }
    Maps tm;
    {
        const cudaError_t e = encode_maps(FMT, codes, scales, n, k, tm);
        if (e != cudaSuccess) return e;
    }
    Params prm = {};
    prm.x = x;
    prm.y = y;
    prm.n = n;
    prm.k = k;
    prm.batch = batch;
    prm.y_dtype = y_dtype;
    prm.stages = pl.stages;
    prm.row_tiles = pl.row_tiles;
    prm.slots = pl.slots;
    prm.slot_bytes = pl.slot_bytes;
    prm.scales_off = pl.scales_off;
    prm.chunk_cap = pl.chunk_cap;
    prm.x_off = pl.x_off;
    prm.red_off = pl.red_off;
    prm.lut_off = pl.lut_off;
    prm.bar_off = pl.bar_off;
    prm.pair_tiles = 0;
    prm.stg_off = 0;
    prm.status = device_status_ptr();
    if (!prm.status) return cudaErrorUnknown;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.grid);
    cfg.blockDim = dim3(threads_of<16>());
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = s;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, gemv_wide_kernel<FMT, NTW, CAP>, tm, prm);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// The kernel is built per largest chunk (2: chunks of 2 and 1 tiles; 4: 4, 2,
// 1; 8: every chunk shape), as the row-owning kernel is.
template <int FMT>
cudaError_t launch_wide_fmt(const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k, const uint16_t* x,
                            int batch, void* y, int y_dtype, const Plan& pl, cudaStream_t s) {
    if (pl.chunk_cap <= 2)
        return pl.nt == 1 ? launch_wide_typed<FMT, 1, 2>(codes, scales, n, k, x, batch, y, y_dtype, pl, s)
                          : launch_wide_typed<FMT, 2, 2>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
    if (pl.chunk_cap <= 4)
        return pl.nt == 1 ? launch_wide_typed<FMT, 1, 4>(codes, scales, n, k, x, batch, y, y_dtype, pl, s)
                          : launch_wide_typed<FMT, 2, 4>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
    return pl.nt == 1 ? launch_wide_typed<FMT, 1, 8>(codes, scales, n, k, x, batch, y, y_dtype, pl, s)
                      : launch_wide_typed<FMT, 2, 8>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
}

}  // namespace rows

bool gemv_wide_eligible(int fmt, int64_t n, int64_t k, int batch) {
    rows::Plan pl;
    return rows::wide_plan(pl, fmt, n, k, batch);
}

cudaError_t launch_gemv_wide(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                             const uint16_t* x, int batch, void* y, int y_dtype, cudaStream_t s) {
    rows::Plan pl;
    if (!rows::wide_plan(pl, fmt, n, k, batch)) return cudaErrorInvalidValue;
    if (fmt == BQ_Q1G128)
        return rows::launch_wide_fmt<BQ_Q1G128>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
    if (fmt == BQ_T2G128) return rows::launch_wide_fmt<BQ_T2G128>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
    return rows::launch_wide_fmt<BQ_T5P8G128>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
}



namespace rows {

// One shared-memory layout for every step: x area for the largest K, 16
// compute warps, one CTA per SM, chunk bound and slot size as a single call
// of the format and batch would use them at one CTA per SM.
bool chain_plan(Plan& pl, int fmt, const bq_chain_step* steps, int nsteps, int batch) {
    int64_t kmax = 0;
    for (int i = 0; i < nsteps; ++i) kmax = steps[i].k > kmax ? steps[i].k : kmax;
    pl.nt = batch <= 2 ? 1 : batch <= 4 ? 2 : 4;
    pl.lanes = batch == 1 ? 16 : 32;
    pl.stages = (int)(kmax / 1024);
    pl.nw = 16;
    const int sms = sm_count();
    pl.grid = sms;
    const int64_t tile_bytes = (fmt == BQ_Q1G128 ? 2048 : fmt == BQ_T2G128 ? 4096 : 16 * kT5RowBytes) + kTileScaleBytes;
    pl.chunk_cap = kMaxChunkTiles;
    const int64_t slot = (pl.chunk_cap * tile_bytes + 1023) / 1024 * 1024;
    pl.slot_bytes = (int)slot;
    pl.scales_off = pl.chunk_cap * (int)(tile_bytes - kTileScaleBytes);
    const int64_t lut = fmt == BQ_T5P8G128 ? kLutBytes : 0;
    const int64_t x_area = ((int64_t)pl.stages * pl.nt * x_nt_bytes(pl.lanes) + 1023) / 1024 * 1024;
    const int64_t red = (int64_t)16 * 32 * pl.nt * 2 * 4;
    const int64_t fixed = 1024 + x_area + red + kChainStgBytes + lut + 2 * kMaxSlots * 8 + 16;
    int64_t slots = (kSmemFull - fixed) / slot;
    if (slots > kMaxSlots) slots = kMaxSlots;
    if (slots < 2) return false;
    pl.slots = (int)slots;
    pl.x_off = (uint32_t)(slots * slot);
    pl.red_off = (uint32_t)(pl.x_off + x_area);
    pl.lut_off = (uint32_t)(pl.red_off + red + kChainStgBytes);  // staging after red
    pl.bar_off = (uint32_t)(pl.lut_off + lut);
    pl.smem = (uint32_t)(1024 + pl.bar_off + 2 * kMaxSlots * 8 + 16);
    pl.ok = true;
    return true;
}

cudaError_t encode_maps(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k, Maps& tm) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    const int64_t row_bytes = (fmt == BQ_Q1G128) ? k / 8 : (fmt == BQ_T2G128) ? k / 4 : (k / 128) * 26;
    const int64_t G = k / 128;
    for (int v = 0; v < 2; ++v) {
        const cuuint32_t rows = v == 0 ? 16u : 128u;
        cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)n};
        cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
        cuuint32_t box[2] = {fmt == BQ_T5P8G128 ? (cuuint32_t)kT5RowBytes : 128u, rows};
        cuuint32_t es[2] = {1, 1};
        if (enc(v == 0 ? &tm.codes16 : &tm.codes128, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims,
                strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                fmt == BQ_T5P8G128 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
        cuuint64_t sdims[2] = {(cuuint64_t)G, (cuuint64_t)n};
        cuuint64_t sstrides[1] = {(cuuint64_t)(G * 2)};
        cuuint32_t sbox[2] = {(cuuint32_t)kGroupsPerStage, rows};
        if (enc(v == 0 ? &tm.scales16 : &tm.scales128, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint16_t*>(scales),
                sdims, sstrides, sbox, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    return cudaSuccess;
}

template <int FMT, int NT, int LANES>
cudaError_t launch_chain_typed(const bq_chain_step* steps, int nsteps, int batch, unsigned int* bar, const Plan& pl,
                               cudaStream_t s) {
    {
        const cudaError_t e =
            ensure_dynamic_smem(reinterpret_cast<const void*>(gemv_chain_kernel<FMT, NT, LANES>), kSmemFull);
        if (e != cudaSuccess) return e;
    }
    ChainMaps tm;
    ChainParams cp;
    cp.nsteps = nsteps;
    cp.bar = bar;
    int* status = device_status_ptr();
    if (!status) return cudaErrorUnknown;
    for (int i = 0; i < nsteps; ++i) {
        const bq_chain_step& st = steps[i];
        const cudaError_t e = encode_maps(FMT, st.codes, st.scales, st.n, st.k, tm.m[i]);
        if (e != cudaSuccess) return e;
        Params& p = cp.step[i];
        p.x = st.x;
        p.y = st.y;
        p.k = st.k;
        p.batch = batch;
        p.y_dtype = st.swiglu ? BQ_BF16 : st.y_dtype;
        p.stages = (int)(st.k / 1024);
        p.pair_tiles = st.swiglu ? (int)(st.n / 2 / 16) : 0;
        p.n = st.swiglu ? st.n / 2 : st.n;  // outputs per batch row
        p.row_tiles = st.swiglu ? p.pair_tiles : (int)((st.n + 15) / 16);
        p.slots = pl.slots;
        p.slot_bytes = pl.slot_bytes;
        p.scales_off = pl.scales_off;
        p.chunk_cap = pl.chunk_cap;
        p.x_off = pl.x_off;
        p.red_off = pl.red_off;
        p.stg_off = pl.red_off + (uint32_t)(16 * 32 * pl.nt * 2 * 4);
        p.lut_off = pl.lut_off;
        p.bar_off = pl.bar_off;
        p.status = status;
    }
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeCooperative;
    attr[1].val.cooperative = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.grid);
    cfg.blockDim = dim3(threads_of<16>());
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, gemv_chain_kernel<FMT, NT, LANES>, tm, cp);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int FMT>
cudaError_t launch_chain_fmt(const bq_chain_step* steps, int nsteps, int batch, unsigned int* bar, const Plan& pl,
                             cudaStream_t s) {
    if (batch == 1) return launch_chain_typed<FMT, 1, 16>(steps, nsteps, batch, bar, pl, s);
    if (pl.nt == 1) return launch_chain_typed<FMT, 1, 32>(steps, nsteps, batch, bar, pl, s);
    if (pl.nt == 2) return launch_chain_typed<FMT, 2, 32>(steps, nsteps, batch, bar, pl, s);
    return launch_chain_typed<FMT, 4, 32>(steps, nsteps, batch, bar, pl, s);
}

}  // namespace rows

bool gemv_chain_eligible(int fmt, const bq_chain_step* steps, int nsteps, int batch) {
    if (fmt != BQ_Q1G128 && fmt != BQ_T2G128 && fmt != BQ_T5P8G128) return false;
    if (nsteps < 1 || nsteps > rows::kMaxChainSteps || batch < 1 || batch > 8) return false;
    for (int i = 0; i < nsteps; ++i) {
        const bq_chain_step& st = steps[i];
        if (st.k <= 0 || st.k % 1024 != 0 || st.k > ((int64_t)1 << 20) || st.n <= 0 || st.n > (int64_t)INT32_MAX - 16)
            return false;
        if (st.swiglu && (st.n % 32 != 0)) return false;  // whole gate and up row tiles
    }
    rows::Plan pl;
    return rows::chain_plan(pl, fmt, steps, nsteps, batch);
}

cudaError_t launch_gemv_chain(int fmt, const bq_chain_step* steps, int nsteps, int batch, unsigned int* bar,
                              cudaStream_t s) {
    rows::Plan pl;
    if (!rows::chain_plan(pl, fmt, steps, nsteps, batch)) return cudaErrorInvalidValue;
    if (fmt == BQ_Q1G128) return rows::launch_chain_fmt<BQ_Q1G128>(steps, nsteps, batch, bar, pl, s);
    if (fmt == BQ_T2G128) return rows::launch_chain_fmt<BQ_T2G128>(steps, nsteps, batch, bar, pl, s);
    return rows::launch_chain_fmt<BQ_T5P8G128>(steps, nsteps, batch, bar, pl, s);
}


cudaError_t launch_gemv_rows(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                             const uint16_t* x, int batch, void* y, int y_dtype, cudaStream_t s) {
    const rows::Plan pl = rows::make_plan(fmt, n, k, batch);
    if (!pl.ok) return cudaErrorInvalidValue;
    if (fmt == BQ_Q1G128) return rows::launch_fmt<BQ_Q1G128>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
    if (fmt == BQ_A1G128) return rows::launch_fmt<BQ_A1G128>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
    if (fmt == BQ_T2G128) return rows::launch_fmt<BQ_T2G128>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
    return rows::launch_fmt<BQ_T5P8G128>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
}

}  // namespace bq
