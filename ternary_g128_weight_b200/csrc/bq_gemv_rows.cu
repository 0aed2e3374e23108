// Decode GEMV, one launch per call: each CTA owns a contiguous range of whole
// weight rows and reduces over all of K itself, so there is no workspace, no
// preparation kernel and no cross-CTA reduction (binary g128, 2-bit-slot and
// 5-trits-per-byte ternary g128, batch 1..8, K % 1024 == 0, while the
// activation operand of all of K fits in shared memory).
//
// Arithmetic (as in the split-K tensor-core GEMV): the codes are expanded with
// one LOP3 per four weights into int8 operands of the warp MMA m16n8k32,
//   binary : byte j of (w & (0x01010101 << p)) = 2^p * bit(8j+p),
//   2-bit  : byte j of (w & (0x03030303 << 2i)) = 4^i * c(4j+i), c = q+1,
//   5-trit : a byte v = sum c_i 3^i ("把 27B 模型压到 4GB" section 2.4: 3^5 <= 256)
//            gives c0..c3 as the four bytes of a 256-entry table word (one
//            copy per lane in shared memory, so lookups never conflict) and
//            c4 = (810 v) >> 16 (exact for v < 243),
// against activations in per-(batch row, group) fixed point Q (largest |x| of
// the group mapped into [2^29, 2^30), Q a multiple of 2^7 resp. 2^6), split
// into four signed base-256 digits, one MMA column each; the k-slot of class
// p (i) carries Q / 2^p (Q / 4^i), so every product is bit * Q or c * Q
// exactly.  Per group and row the int32 column sums are recombined in FP32:
//   binary : y += s * (2 * 2^-E * sum bit Q - 2^-E * sum Q)
//   ternary: y += s * (    2^-E * sum c   Q - 2^-E * sum Q)
// ("Bonsai-27B ... Binary g128": 0 -> -scale, 1 -> +scale; "1-bit Bonsai 8B"
// notes, section 4.1: one FP16 scale per 128 weights).
//
// CTA (one per SM): 16 compute warps and one producer warp.
//   * The producer streams the CTA's weights -- per (chunk of up to 8 row
//     tiles of 16 rows, stage of 1024 K) TMA boxes of codes (128-byte
//     swizzle) and scales -- into a ring of shared-memory slots, starting
//     before the wait on the previous kernel in the stream (programmatic
//     dependent launch): the weights do not depend on it.  A full chunk is
//     one 128-row box per 128-byte column (one TMA instruction per 16 KB:
//     with one box per 16-row tile the TMA issue, not HBM, limited the
//     stream to ~43% of the HBM bandwidth); a partial chunk uses 16-row boxes.
//   * After that wait the compute warps turn x into the MMA B fragments and
//     the per-group recombination table for all of K, once per CTA, into
//     shared memory.
//   * A chunk of CT row tiles (CT = 8, 4, 2 or 1) gives each row tile
//     16/CT warps (at most 8), each taking an equal share of the stage's 8
//     groups; the warps sharing a row tile add their partial sums through
//     shared memory in warp order (deterministic).
#include <cuda.h>

#include "bq_internal.cuh"
#include "bq_ptx.cuh"

namespace bq {
namespace rows {

constexpr int kGroupsPerStage = 8;  // 1024 K per stage
constexpr int kComputeWarps = 16;
constexpr int kProducerWarp = kComputeWarps;
constexpr int kThreads = (kComputeWarps + 1) * 32;
constexpr int kMaxChunkTiles = 8;  // chunk bound of the 2-bit and 5-trit formats
constexpr int kTileScaleBytes = 16 * kGroupsPerStage * 2;  // 256
constexpr int kMaxSlots = 8;
constexpr int kSmemLimit = 232448;  // opt-in shared memory per block on sm_100
constexpr uint32_t kWaitPolls = 1u << 23;

template <int FMT>
struct Fmt;
template <>
struct Fmt<BQ_Q1G128> {
    static constexpr int kBoxes = 1;         // 128-byte columns per row tile and stage
    static constexpr int kCoefShift = 1;     // 2 * sum(bit * x) - sum(x)
    static constexpr int kQuantShift = 7;    // Q multiple of 2^7
};
template <>
struct Fmt<BQ_T2G128> {
    static constexpr int kBoxes = 2;
    static constexpr int kCoefShift = 0;     // sum(c * x) - sum(x)
    static constexpr int kQuantShift = 6;    // Q multiple of 2^6
};
template <>
struct Fmt<BQ_T5P8G128> {
    static constexpr int kBoxes = 1;         // one unswizzled 208-byte column (8 groups x 26 bytes)
    static constexpr int kCoefShift = 0;     // sum(c * x) - sum(x)
    static constexpr int kQuantShift = 0;    // plain bytes c, operand Q
};
constexpr int kT5RowBytes = kGroupsPerStage * 26;  // 208
constexpr int kLutBytes = 256 * 32 * 4;           // byte -> c0..c3, one copy per lane
// Slot layout: codes [column box b][row tile i][16 rows][128 B] (so that a
// 128-row box of column b lands on all 8 row tiles at once; 5-trit format:
// [row tile i][16 rows][208 B]), then scales [row tile i][16 rows][8 groups]
// FP16.
template <int FMT>
constexpr int tile_code_bytes() { return FMT == BQ_T5P8G128 ? 16 * kT5RowBytes : Fmt<FMT>::kBoxes * 16 * 128; }
constexpr int kBoxColumnBytes = kMaxChunkTiles * 16 * 128;  // 16 KB
// Row tiles per chunk the kernel is built for: 16 for the binary format up
// to batch 4 (each of the 16 compute warps then owns one row tile and all 8
// groups of a stage), else 8; a call uses 16 only where a CTA owns at least
// 16 row tiles (see make_plan).
template <int FMT, int NT>
constexpr int mct() { return (FMT == BQ_Q1G128 && NT <= 2) ? 16 : kMaxChunkTiles; }


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
    int chunk_cap;      // row tiles per chunk, at most (8, or 16 for binary)
    uint32_t x_off, red_off, lut_off, bar_off;  // shared-memory offsets
    int* status;
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

__device__ __forceinline__ void bar_compute() { asm volatile("bar.sync 1, %0;" ::"n"(kComputeWarps * 32) : "memory"); }

__device__ __forceinline__ int chunk_tiles(int remaining, int cap) {
    return (cap >= 16 && remaining >= 16) ? 16 : remaining >= 8 ? 8 : remaining >= 4 ? 4 : remaining >= 2 ? 2 : 1;
}

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
// Warp-wide: group G of stage st for all n-tiles.  Lane l holds k = 4l .. 4l+3
// of the group.  The byte of digit d of batch row bb for weight k goes to the
// B fragment of lane (4 (d + 4 (bb & 1)) + t), MMA q, register h, byte j,
// where (t, q, h, j) is the k-slot the A decode gives weight k:
//   binary: k = 32t + 8j + 2q + h   (word t of the row's group, class 2q+h)
//   2-bit : k = 32t + 16h + 4j + q  (word 2t+h of the row's group, class q)
//   5-trit: A register i = 2q + h of thread t holds, for i < 6, digits 0..3
//           of byte 6t+i; i = 6 digit 4 of bytes 6t..6t+3; i = 7 digit 4 of
//           bytes 6t+4, 6t+5 and trits 120+2t, 121+2t (the group's last
//           eight trits, in bytes 24 and 25)
// Table entry (G, t) of an n-tile, t = 2 (bb & 1) + hh for digit pair hh, with
// e = coef - E + 16 hh and z = [hh == 0] 2^-E sum Q:
//   one factor  : {2^e, 1, z, 0}, u = (D0 + 256 D1) 2^e - z;
//   two factors : {2^a, 2^(e-a), z, 1} when 2^e is not a normal float,
//                 u = (D0 + 256 D1) 2^a 2^(e-a) - z.
// Rows past the batch get zero entries with the group's flag (so that the
// kernel's choice stays uniform across the warp).
// This lane's 4 BF16 activations of group G of stage st for the batch rows of
// the n-tiles (zero past the batch).
template <int NT>
__device__ __forceinline__ void load_group_x(const Params& p, int st, int G, int lane, uint2 (&raw)[2 * NT]) {
    const int64_t kbase = (int64_t)st * 1024 + G * 128;
#pragma unroll
    for (int bb = 0; bb < 2 * NT; ++bb)
        raw[bb] = bb < p.batch ? __ldg(reinterpret_cast<const uint2*>(p.x + bb * p.k + kbase + lane * 4))
                               : make_uint2(0u, 0u);
}

template <int FMT, int NT, int LANES>
__device__ void prep_group(const Params& p, uint8_t* xst, int G, int lane, const uint2 (&xraw)[2 * NT]) {
    constexpr int X_NT = x_nt_bytes(LANES);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        uint8_t* xt = xst + nt * X_NT;
        float xv[2][4];
        int E[2];
        bool two = false;
#pragma unroll
        for (int hb = 0; hb < 2; ++hb) {
            const uint2 raw = xraw[2 * nt + hb];
            xv[hb][0] = bf16_lo(raw.x);
            xv[hb][1] = bf16_hi(raw.x);
            xv[hb][2] = bf16_lo(raw.y);
            xv[hb][3] = bf16_hi(raw.y);
            E[hb] = 0;
            if (2 * nt + hb < p.batch) {  // (warp-uniform)
                float m = fmaxf(fmaxf(fabsf(xv[hb][0]), fabsf(xv[hb][1])), fmaxf(fabsf(xv[hb][2]), fabsf(xv[hb][3])));
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
                E[hb] = (m > 0.f) ? 29 - ilog2f(m) : 0;
                if (Fmt<FMT>::kCoefShift - E[hb] < -126) two = true;
            }
        }
#pragma unroll
        for (int hb = 0; hb < 2; ++hb) {
            const int bb = 2 * nt + hb;
            float4* tabp = reinterpret_cast<float4*>(xt + kGroupsPerStage * 2 * LANES * 16) + G * 4 + 2 * hb;
            if (bb >= p.batch) {
                // zero digits (rows of a 32-lane tile) and zero table entries
                if (LANES == 32) {
                    const int ln0 = 4 * (4 * hb) + (lane & 3), pp = (lane >> 2) & 1, dd = lane >> 3;
                    *reinterpret_cast<uint4*>(xt + ((G * 2 + pp) * LANES + ln0 + 4 * dd) * 16) = make_uint4(0u, 0u, 0u, 0u);
                }
                if (lane < 2) tabp[lane] = make_float4(0.0f, 0.0f, 0.0f, two ? 1.0f : 0.0f);
                continue;
            }
            const int es = E[hb] - Fmt<FMT>::kQuantShift;  // x * 2^es -> Q / 2^shift
            const int e1 = max(-126, min(127, es));
            const float p1 = exp2i(e1), p2 = exp2i(es - e1);
            long long sumq = 0;
            // (k-slot of this lane's first value; the others differ by compile-time offsets)
            uint8_t* xb = xt + (G * 2) * LANES * 16;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int kk = lane * 4 + i;
                const int Q = __float2int_rn(xv[hb][i] * p1 * p2) << Fmt<FMT>::kQuantShift;
                sumq += Q;
                int b, t, q, h, j;
                if (FMT == BQ_Q1G128) {
                    b = Q >> (kk & 7);  // exact: Q is a multiple of 2^7
                    t = kk >> 5; j = (kk >> 3) & 3; q = (kk >> 1) & 3; h = kk & 1;
                } else if (FMT == BQ_T2G128) {
                    b = Q >> (2 * (kk & 3));  // exact: Q is a multiple of 2^6
                    t = kk >> 5; h = (kk >> 4) & 1; j = (kk >> 2) & 3; q = kk & 3;
                } else {
                    b = Q;
                    int ri;  // A register of the thread
                    if (kk < 120) {
                        const int byte = kk / 5, d = kk - 5 * byte, ib = byte % 6;
                        t = byte / 6;
                        if (d < 4) { ri = ib; j = d; }
                        else if (ib < 4) { ri = 6; j = ib; }
                        else { ri = 7; j = ib - 4; }
                    } else {
                        const int e = kk - 120;
                        t = e >> 1; ri = 7; j = 2 + (e & 1);
                    }
                    q = ri >> 1; h = ri & 1;
                }
                // balanced base-256 digits d0..d3 of b (|b| < 2^30): the bytes of
                // (b + 0x808080) ^ 0x808080 (adding 128 to the three low digits
                // keeps every byte in [0, 255], so no carry crosses a byte)
                const uint32_t w = ((uint32_t)b + 0x808080u) ^ 0x808080u;
                uint8_t* dst = xb + ((q >> 1) * LANES + 4 * (4 * hb) + t) * 16 + (q & 1) * 8 + h * 4 + j;
#pragma unroll
                for (int d = 0; d < 4; ++d) dst[d * 4 * 16] = (uint8_t)(w >> (8 * d));  // lane 4 (d + 4 hb) + t
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) sumq += __shfl_xor_sync(0xffffffffu, sumq, off);
            if (lane < 2) {
                const int hh = lane;  // digit pair (0,1) or (2,3)
                const int e = Fmt<FMT>::kCoefShift - E[hb] + 16 * hh;
                const double z = (hh == 0) ? ldexp((double)sumq, -E[hb]) : 0.0;
                const int a = two ? max(-60, min(60, e)) : e;
                float4 tab;
                tab.x = exp2i(a);
                tab.y = exp2i(e - a);
                tab.z = (float)z;
                tab.w = two ? 1.0f : 0.0f;
                tabp[hh] = tab;
            }
        }
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

// ------------------------------------------------------------ one chunk
// CT row tiles (16 rows each) starting at row tile rt, all stages.  Warp w
// takes row tile w / WPR and groups G = w % WPR + WPR i (i < 8 / WPR), with
// WPR = min(16 / CT, 8) warps per row tile; warps past CT row tiles only
// keep the stage barriers going.
template <int FMT, int NT, int LANES, int CT>
__device__ bool run_chunk(const Params& p, uint8_t* smem, uint64_t* full, uint64_t* empty, int rt, Ring& rp,
                          int warp, int lane) {
    constexpr int WPR = (kComputeWarps / CT) < kGroupsPerStage ? (kComputeWarps / CT) : kGroupsPerStage;
    constexpr int GPW = kGroupsPerStage / WPR;  // groups per warp and stage
    constexpr int TCB = tile_code_bytes<FMT>();
    constexpr int X_NT = x_nt_bytes(LANES);
    const int my_rt = warp / WPR, gsub = warp % WPR;
    const bool active = my_rt < CT;
    const int g = lane >> 2, t = lane & 3;
    // at batch 1 the upper 16 lanes (columns of a second batch row) read the
    // lower lanes' fragments: their sums are never stored
    const int blane = lane & (LANES - 1);
    const uint8_t* xres = smem + p.x_off;
    const uint32_t* lut = reinterpret_cast<const uint32_t*>(smem + p.lut_off);
    const uint32_t t5sel = (uint32_t)(2 * t) | ((uint32_t)(2 * t + 1) << 4);
    float yacc[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) yacc[nt][0] = yacc[nt][1] = 0.0f;
    bool alive = true;
    for (int st = 0; st < p.stages; ++st, rp.next()) {
        const int slot = rp.slot;
        if (!ptx::mbar_wait_bounded(&full[slot], rp.round & 1u, kWaitPolls)) {
            record_status(p.status, BQ_ERR_TIMEOUT);
            alive = false;
            break;
        }
        if (!active) {
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&empty[slot]);
            continue;
        }
        const uint8_t* sb = smem + slot * p.slot_bytes;
        const uint8_t* codes_t = sb + my_rt * 2048;  // column box 0 of this row tile
        const uint16_t* scales_t = reinterpret_cast<const uint16_t*>(sb + p.scales_off + my_rt * kTileScaleBytes);
        const uint8_t* xs = xres + (size_t)st * NT * X_NT;
#pragma unroll
        for (int gi = 0; gi < GPW; ++gi) {
            const int G = gsub + WPR * gi;
            uint4 bf[NT][2];
            float4 tab[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const uint8_t* xt = xs + nt * X_NT;
#pragma unroll
                for (int h = 0; h < 2; ++h) bf[nt][h] = *reinterpret_cast<const uint4*>(xt + ((G * 2 + h) * LANES + blane) * 16);
                tab[nt] = *reinterpret_cast<const float4*>(xt + kGroupsPerStage * 2 * LANES * 16 + (G * 4 + t) * 16);
            }
            int acc[NT][4];
            if (FMT == BQ_Q1G128) {
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
                const uint8_t* g0 = sb + my_rt * TCB + g * kT5RowBytes + 26 * G;
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
                const uint8_t* box = codes_t + (G >> 2) * kBoxColumnBytes;
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
            const float s0 = half_bits_to_float(scales_t[g * kGroupsPerStage + G]);
            const float s1 = half_bits_to_float(scales_t[(g + 8) * kGroupsPerStage + G]);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                // D0 + 256 D1 is exact in int32 (|D0|, |D1| <= 2^21)
                const float v0 = (float)(acc[nt][0] + (acc[nt][1] << 8));
                const float v1 = (float)(acc[nt][2] + (acc[nt][3] << 8));
                // (with one factor tab.y = 1: the same rounding as fmaf(v, 2^e, -z))
                const float u0 = fmaf(v0 * tab[nt].x, tab[nt].y, -tab[nt].z);
                const float u1 = fmaf(v1 * tab[nt].x, tab[nt].y, -tab[nt].z);
                yacc[nt][0] = fmaf(s0, u0, yacc[nt][0]);
                yacc[nt][1] = fmaf(s1, u1, yacc[nt][1]);
            }
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&empty[slot]);
    }
    // digit pairs (t, t^1) -> one value per (batch row, row) on even t
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int r = 0; r < 2; ++r) yacc[nt][r] += __shfl_xor_sync(0xffffffffu, yacc[nt][r], 1);
    if (WPR > 1) {
        // partial sums of the warps sharing a row tile, added in warp order
        float* red = reinterpret_cast<float*>(smem + p.red_off);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int r = 0; r < 2; ++r) red[((warp * 32 + lane) * NT + nt) * 2 + r] = yacc[nt][r];
        bar_compute();
        if (active && gsub == 0) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    float s = 0.0f;
#pragma unroll
                    for (int j = 0; j < WPR; ++j) s += red[(((warp + j) * 32 + lane) * NT + nt) * 2 + r];
                    yacc[nt][r] = s;
                }
        }
        bar_compute();  // red is reused by the next chunk
    }
    if (active && gsub == 0 && (t & 1) == 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int bb = nt * 2 + (t >> 1);
                const int64_t row = (int64_t)(rt + my_rt) * 16 + g + 8 * r;
                if (bb < p.batch && row < p.n) {
                    if (p.y_dtype == BQ_F32)
                        static_cast<float*>(p.y)[bb * p.n + row] = yacc[nt][r];
                    else
                        static_cast<uint16_t*>(p.y)[bb * p.n + row] = float_to_bf16_bits(yacc[nt][r]);
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

template <int FMT, int NT, int LANES>
__global__ void __launch_bounds__(kThreads, 1) gemv_rows_kernel(const __grid_constant__ Maps tm, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = ptx::align_smem<1024>(smem_raw);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.bar_off);
    uint64_t* empty = full + kMaxSlots;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = gridDim.x, c = blockIdx.x;
    const int rt0 = (int)((int64_t)c * p.row_tiles / C), rt1 = (int)((int64_t)(c + 1) * p.row_tiles / C);

    if (threadIdx.x == 0) {
        for (int i = 0; i < p.slots; ++i) {
            ptx::mbar_init(&full[i], 1);
            ptx::mbar_init(&empty[i], kComputeWarps);
        }
        ptx::fence_barrier_init();
    }
    __syncthreads();
    ptx::pdl_launch_dependents();

    if (warp == kProducerWarp) {
        // ------------------------------------------------ weight producer
        if (lane == 0) {
            ptx::prefetch_tensormap(&tm.codes16);
            ptx::prefetch_tensormap(&tm.scales16);
            ptx::prefetch_tensormap(&tm.codes128);
            ptx::prefetch_tensormap(&tm.scales128);
            constexpr int TCB = tile_code_bytes<FMT>();
            int it = 0;
            Ring rp;
            rp.depth = p.slots;
            bool alive = true;
            for (int r = rt0; r < rt1 && alive;) {
                const int ct = chunk_tiles(rt1 - r, p.chunk_cap);
                for (int st = 0; st < p.stages; ++st, ++it, rp.next()) {
                    const int slot = rp.slot;
                    if (rp.round > 0 && !ptx::mbar_wait_bounded(&empty[slot], (rp.round - 1) & 1u, kWaitPolls)) {
                        record_status(p.status, BQ_ERR_TIMEOUT);
                        alive = false;
                        break;
                    }
                    uint8_t* sb = smem + slot * p.slot_bytes;
                    ptx::mbar_arrive_expect_tx(&full[slot], (uint32_t)(ct * (TCB + kTileScaleBytes)));
                    if (FMT == BQ_T5P8G128) {
                        if (ct == kMaxChunkTiles) {
                            ptx::tma_load_2d(sb, &tm.codes128, st * kT5RowBytes, r * 16, &full[slot]);
                            ptx::tma_load_2d(sb + p.scales_off, &tm.scales128, st * kGroupsPerStage, r * 16,
                                             &full[slot]);
                        } else {
                            for (int i = 0; i < ct; ++i) {
                                ptx::tma_load_2d(sb + i * TCB, &tm.codes16, st * kT5RowBytes, (r + i) * 16, &full[slot]);
                                ptx::tma_load_2d(sb + p.scales_off + i * kTileScaleBytes, &tm.scales16,
                                                 st * kGroupsPerStage, (r + i) * 16, &full[slot]);
                            }
                        }
                    } else if (ct >= kMaxChunkTiles) {
                        // 128-row boxes: one per 128-byte column (2-bit) or per 8 row tiles (binary)
                        for (int h8 = 0; h8 < ct / kMaxChunkTiles; ++h8) {
#pragma unroll
                            for (int b = 0; b < Fmt<FMT>::kBoxes; ++b)
                                ptx::tma_load_2d(sb + b * kBoxColumnBytes + h8 * kBoxColumnBytes, &tm.codes128,
                                                 st * (Fmt<FMT>::kBoxes * 128) + b * 128, (r + 8 * h8) * 16, &full[slot]);
                            ptx::tma_load_2d(sb + p.scales_off + h8 * kMaxChunkTiles * kTileScaleBytes,
                                             &tm.scales128, st * kGroupsPerStage, (r + 8 * h8) * 16, &full[slot]);
                        }
                    } else {
                        for (int i = 0; i < ct; ++i) {
#pragma unroll
                            for (int b = 0; b < Fmt<FMT>::kBoxes; ++b)
                                ptx::tma_load_2d(sb + b * kBoxColumnBytes + i * 2048, &tm.codes16,
                                                 st * (Fmt<FMT>::kBoxes * 128) + b * 128, (r + i) * 16, &full[slot]);
                            ptx::tma_load_2d(sb + p.scales_off + i * kTileScaleBytes, &tm.scales16,
                                             st * kGroupsPerStage, (r + i) * 16, &full[slot]);
                        }
                    }
                }
                r += ct;
            }
            // every copy this CTA issued must land before it may exit
            for (int j = (it > p.slots ? it - p.slots : 0); j < it; ++j)
                if (!ptx::mbar_wait_bounded(&full[j % p.slots], (uint32_t)((j / p.slots) & 1), kWaitPolls))
                    record_status(p.status, BQ_ERR_TIMEOUT);
        }
        return;
    }

    // ---------------------------------------------------- compute warps
    if (FMT == BQ_T5P8G128) {
        // digit table: lut[32 v + l] = c0 | c1 << 8 | c2 << 16 | c3 << 24 of byte v
        uint32_t* lut = reinterpret_cast<uint32_t*>(smem + p.lut_off);
        for (int i = threadIdx.x; i < 256 * 32; i += kComputeWarps * 32) {
            const uint32_t v = (uint32_t)i >> 5;
            lut[i] = (v % 3u) | ((v / 3u % 3u) << 8) | ((v / 9u % 3u) << 16) | ((v / 27u % 3u) << 24);
        }
    }
    ptx::pdl_wait();  // x is produced, y may still be read, by the previous kernel
    {
        // items (stage, group) i = warp + 16 j; the x loads of up to kPrepBatch
        // items are issued before any of them is processed
        constexpr int kPrepBatch = 4;
        uint8_t* xres = smem + p.x_off;
        const int items = p.stages * kGroupsPerStage;
        for (int i0 = warp; i0 < items; i0 += kComputeWarps * kPrepBatch) {
            uint2 raw[kPrepBatch][2 * NT];
#pragma unroll
            for (int j = 0; j < kPrepBatch; ++j) {
                const int i = i0 + j * kComputeWarps;
                if (i < items) load_group_x<NT>(p, i / kGroupsPerStage, i % kGroupsPerStage, lane, raw[j]);
            }
#pragma unroll
            for (int j = 0; j < kPrepBatch; ++j) {
                const int i = i0 + j * kComputeWarps;
                if (i < items)
                    prep_group<FMT, NT, LANES>(p, xres + (size_t)(i / kGroupsPerStage) * NT * x_nt_bytes(LANES),
                                               i % kGroupsPerStage, lane, raw[j]);
            }
        }
    }
    bar_compute();
    Ring rp;
    rp.depth = p.slots;
    for (int r = rt0; r < rt1;) {
        const int ct = chunk_tiles(rt1 - r, p.chunk_cap);
        bool ok;
        if (mct<FMT, NT>() >= 16 && ct == 16)
            ok = run_chunk<FMT, NT, LANES, mct<FMT, NT>()>(p, smem, full, empty, r, rp, warp, lane);
        else if (ct == 8)
            ok = run_chunk<FMT, NT, LANES, 8>(p, smem, full, empty, r, rp, warp, lane);
        else if (ct == 4)
            ok = run_chunk<FMT, NT, LANES, 4>(p, smem, full, empty, r, rp, warp, lane);
        else if (ct == 2)
            ok = run_chunk<FMT, NT, LANES, 2>(p, smem, full, empty, r, rp, warp, lane);
        else
            ok = run_chunk<FMT, NT, LANES, 1>(p, smem, full, empty, r, rp, warp, lane);
        if (!ok) break;
        r += ct;
    }
}

// ----------------------------------------------------------------- host
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

int sm_count() {
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
            sms = 148;
    }
    return sms;
}

struct Plan {
    int nt = 0, lanes = 0, stages = 0, row_tiles = 0, slots = 0, grid = 0, chunk_cap = 8, slot_bytes = 0, scales_off = 0;
    uint32_t x_off = 0, red_off = 0, lut_off = 0, bar_off = 0, smem = 0;
    bool ok = false;
};

Plan make_plan(int fmt, int64_t n, int64_t k, int batch) {
    Plan pl;
    if (!((fmt == BQ_Q1G128 || fmt == BQ_T2G128 || fmt == BQ_T5P8G128) && batch >= 1 && batch <= 8 && k > 0 &&
          k % 1024 == 0 && n > 0 &&
          n <= (int64_t)INT32_MAX - 16 && k / 4 <= (int64_t)INT32_MAX / 4 && k <= (int64_t)1 << 20))
        return pl;
    pl.nt = batch <= 2 ? 1 : batch <= 4 ? 2 : 4;  // n-tiles of two batch rows (5..8 -> 4)
    pl.lanes = batch == 1 ? 16 : 32;
    pl.stages = (int)(k / 1024);
    pl.row_tiles = (int)((n + 15) / 16);
    const int sms = sm_count();
    pl.grid = pl.row_tiles < sms ? pl.row_tiles : sms;
    // 16-tile chunks (binary, batch <= 4) only where a CTA owns at least 16
    // row tiles; otherwise 8-tile slots keep the ring deep
    const int64_t tile_bytes = (fmt == BQ_Q1G128 ? 2048 : fmt == BQ_T2G128 ? 4096 : 16 * kT5RowBytes) + kTileScaleBytes;
    pl.chunk_cap = (fmt == BQ_Q1G128 && pl.nt <= 2 && pl.row_tiles / pl.grid >= 16) ? 16 : kMaxChunkTiles;
    const int64_t slot = pl.chunk_cap * tile_bytes;
    pl.slot_bytes = (int)slot;
    pl.scales_off = pl.chunk_cap * (int)(tile_bytes - kTileScaleBytes);
    const int64_t lut = fmt == BQ_T5P8G128 ? kLutBytes : 0;
    const int64_t x_area = ((int64_t)pl.stages * pl.nt * x_nt_bytes(pl.lanes) + 1023) / 1024 * 1024;
    const int64_t red = (int64_t)kComputeWarps * 32 * pl.nt * 2 * 4;
    const int64_t fixed = 1024 + x_area + red + lut + 2 * kMaxSlots * 8;
    int64_t slots = (kSmemLimit - fixed) / slot;
    if (slots > kMaxSlots) slots = kMaxSlots;
    if (slots < 2) return pl;
    pl.slots = (int)slots;
    pl.x_off = (uint32_t)(slots * slot);
    pl.red_off = (uint32_t)(pl.x_off + x_area);
    pl.lut_off = (uint32_t)(pl.red_off + red);
    pl.bar_off = (uint32_t)(pl.lut_off + lut);
    pl.smem = (uint32_t)(1024 + pl.bar_off + 2 * kMaxSlots * 8);
    pl.ok = true;
    return pl;
}

template <int FMT, int NT, int LANES>
cudaError_t launch_typed(const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k, const uint16_t* x,
                         int batch, void* y, int y_dtype, const Plan& pl, cudaStream_t s) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(gemv_rows_kernel<FMT, NT, LANES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kSmemLimit);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const int64_t row_bytes = (FMT == BQ_Q1G128) ? k / 8 : (FMT == BQ_T2G128) ? k / 4 : (k / 128) * 26;
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
            cuuint64_t dims[2] = {(cuuint64_t)G, (cuuint64_t)n};
            cuuint64_t strides[1] = {(cuuint64_t)(G * 2)};
            cuuint32_t box[2] = {(cuuint32_t)kGroupsPerStage, rows};
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
    prm.status = device_status_ptr();
    if (!prm.status) return cudaErrorUnknown;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = s;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, gemv_rows_kernel<FMT, NT, LANES>, tm, prm);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace rows

bool gemv_rows_eligible(int fmt, int64_t n, int64_t k, int batch) { return rows::make_plan(fmt, n, k, batch).ok; }

cudaError_t launch_gemv_rows(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                             const uint16_t* x, int batch, void* y, int y_dtype, cudaStream_t s) {
    const rows::Plan pl = rows::make_plan(fmt, n, k, batch);
    if (!pl.ok) return cudaErrorInvalidValue;
    if (fmt == BQ_Q1G128) {
        if (batch == 1) return rows::launch_typed<BQ_Q1G128, 1, 16>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
        if (pl.nt == 1) return rows::launch_typed<BQ_Q1G128, 1, 32>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
        if (pl.nt == 2) return rows::launch_typed<BQ_Q1G128, 2, 32>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
        return rows::launch_typed<BQ_Q1G128, 4, 32>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
    }
    if (fmt == BQ_T2G128) {
        if (batch == 1) return rows::launch_typed<BQ_T2G128, 1, 16>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
        if (pl.nt == 1) return rows::launch_typed<BQ_T2G128, 1, 32>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
        if (pl.nt == 2) return rows::launch_typed<BQ_T2G128, 2, 32>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
        return rows::launch_typed<BQ_T2G128, 4, 32>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
    }
    if (batch == 1) return rows::launch_typed<BQ_T5P8G128, 1, 16>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
    if (pl.nt == 1) return rows::launch_typed<BQ_T5P8G128, 1, 32>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
    if (pl.nt == 2) return rows::launch_typed<BQ_T5P8G128, 2, 32>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
    return rows::launch_typed<BQ_T5P8G128, 4, 32>(codes, scales, n, k, x, batch, y, y_dtype, pl, s);
}

}  // namespace bq
