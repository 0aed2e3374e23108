// Prefill GEMM on the 5th-generation tensor cores: Y[t][r] = sum_k X[t][k] *
// s[r][g(k)] q[r][k] for T tokens ("1-bit Bonsai 8B" notes, summary section 3
// and Table 3 pp512: prompt processing is a dense contraction).
//
// Operands.  W tiles are dequantised on chip to FP16 s*q -- exact, since s is
// FP16 and q is -1, 0 or +1 -- and never written to global memory.  X is
// converted once per call to FP16 with a per-token power-of-two pre-scale
// 2^e_t that maps the token's largest |x| into [2^14, 2^15): every BF16 value
// within 2^-31 of that largest magnitude converts exactly (BF16 has 8
// significant bits, FP16 11 bits down to 2^-24).  The tensor core accumulates
// in FP32 and the epilogue multiplies by 2^-e_t (exact) before rounding to
// BF16.
//
// K order.  Inside each 64-wide K stage the FP16 operand rows are stored in a
// permuted order (kperm below) chosen so that the packed codes expand into
// FP16 pairs with two to four integer / half2 operations and no selects: the
// binary format pairs bits m and m+16 of a 32-bit code word, the 2-bit format
// codes m and m+8 of a word, the base-3 format the same digit of two bytes
// held in the two 16-bit halves of one register.  X' is written in the same
// order, so the contraction over the stage is unchanged.
//
// CTA (one per SM, persistent).  Tile = 128 weight rows x tile_n tokens
// (tile_n = T rounded up to 32, at most 256), K in stages of 64 (one 128-byte
// swizzle row of FP16).  When the row tiles alone cannot fill the GPU, each
// tile's K range is split over several CTAs and a second kernel adds the FP32
// partial tiles in a fixed order.
//   dequant warps (8 binary, 12 ternary): dequantise the tile's 128 weight
//                rows into the stage's A buffer (K-major, 128-byte swizzle,
//                the UMMA canonical layout), two or three sets of four warps
//                taking the stages in turn, packed codes fetched four of
//                their stages ahead;
//   next warp  : TMA loads of the FP16 activation tile (same layout) into B;
//   next warp  : allocates TMEM (2 x 256 columns) and issues
//                tcgen05.mma.kind::f16 (M = 128, N = tile_n, K = 16);
//   last 4     : epilogue: TMEM -> registers -> Y (or the partial tile), while
//                the MMAs of the next work unit accumulate in the other buffer
//                (warp w reads TMEM lane quadrant w % 4).
// Work units are taken token-tile-major so that the activation tile in flight
// and the packed weights stay resident in L2.
#include <cuda.h>

#include "bq_internal.cuh"
#include "bq_ptx.cuh"

namespace bq {
namespace gemm {

constexpr int kTileM = 128;      // weight rows
constexpr int kMaxTileN = 256;   // tokens
constexpr int kStageK = 64;      // FP16 K per stage = 128 bytes per row
constexpr int kStages = 4;
constexpr int kABytes = kTileM * kStageK * 2;     // 16 KB
constexpr int kBBytes = kMaxTileN * kStageK * 2;  // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
// Sets of 4 dequant warps take the stages in turn: two for the binary
// format, three for the ternary formats, whose decode costs more instructions
// per weight (measured on B200 at T = 4096: the third set took the 5-trit
// GEMM from 0.44 to 0.47 of the BF16 peak on 17408 x 5120 and the 2-bit one
// from 0.59 to 0.60, while it slowed the binary one).
constexpr int kDequantSetWarps = 4, kEpiWarps = 4;
template <int FMT>
struct Roles {
    static constexpr int kSets = FMT == BQ_Q1G128 ? 2 : 3;
    static constexpr int kDequantWarps = kSets * kDequantSetWarps;
    static constexpr int kTmaWarp = kDequantWarps, kMmaWarp = kTmaWarp + 1, kEpiWarp0 = kMmaWarp + 1;
    static constexpr int kThreads = (kEpiWarp0 + kEpiWarps) * 32;
};
constexpr int kTmemCols = 2 * kMaxTileN;
constexpr int kBarriers = 3 * kStages + 4;
constexpr int kSmemBytes = kStages * kStageBytes + 1024 + kBarriers * 8 + 16;
constexpr uint32_t kWaitPolls = 1u << 24;
constexpr int kAhead = 4;  // stages of packed codes in flight per dequant thread

struct Params {
    const uint8_t* codes;
    const uint16_t* scales;
    const float* inv_scale;  // [T] 2^-e_t
    void* y;                 // [T][N] BF16 or FP32 (splits == 1)
    int y_f32;               // output type: FP32 (1) or BF16 (0)
    float* partial;          // [splits][T][N] FP32 sums without the 2^-e_t factor (splits > 1)
    int64_t n, k, t;
    int64_t units;           // row tiles x token tiles x splits
    int tile_n;              // tokens per tile, multiple of 32, <= 256
    int splits;              // K splits per tile
    int* status;
};

// ------------------------------------------------------------ K permutation
// Position p (0..63) of a stage's FP16 row holds K offset kperm(p) of that
// stage; H is the stage's half of its 128-group (only the base-3 format,
// whose byte boundaries differ between the halves, depends on it).
template <int FMT, int H>
__host__ __device__ constexpr int kperm(int p) {
    const int i = p >> 1, b = p & 1;
    if (FMT == BQ_Q1G128) return 32 * (i >> 4) + 16 * b + (i & 15);
    if (FMT == BQ_T2G128) return 16 * (i >> 3) + 8 * b + (i & 7);
    if (H == 0) return i < 30 ? i + 30 * b : 60 + 2 * (i - 30) + b;
    return i < 30 ? 1 + i + 30 * b : (i == 30 ? (b ? 61 : 0) : 62 + b);
}

template <int FMT, int H>
__device__ __forceinline__ void permute_stage(const uint32_t (&in)[32], uint32_t (&out)[32]) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int a = kperm<FMT, H>(2 * i), b = kperm<FMT, H>(2 * i + 1);
        const uint32_t lo = (in[a >> 1] >> (16 * (a & 1))) & 0xFFFFu;
        const uint32_t hi = (in[b >> 1] >> (16 * (b & 1))) & 0xFFFFu;
        out[i] = lo | (hi << 16);
    }
}

// ----------------------------------------------------------------- X prep
// One CTA per token: X' = FP16(x * 2^e) in the permuted K order,
// inv_scale = 2^-e with e = 14 - floor(log2 max|x|) (0 for an all-zero row):
// exact for every BF16 value within 2^-31 of the row's largest magnitude.
template <int FMT>
__global__ void __launch_bounds__(128) xprep_f16_kernel(const uint16_t* __restrict__ x, int64_t k,
                                                        uint16_t* __restrict__ xh, float* __restrict__ inv_scale) {
    __shared__ float s_max[4];
    ptx::pdl_launch_dependents();
    ptx::pdl_wait();
    const int64_t t = blockIdx.x;
    const uint16_t* row = x + t * k;
    float m = 0.0f;
    for (int64_t i = threadIdx.x * 8; i < k; i += blockDim.x * 8) {
        const uint4 v = *reinterpret_cast<const uint4*>(row + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) m = fmaxf(m, fmaxf(fabsf(bf16_lo(w[j])), fabsf(bf16_hi(w[j]))));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((threadIdx.x & 31) == 0) s_max[threadIdx.x >> 5] = m;
    __syncthreads();
    m = fmaxf(fmaxf(s_max[0], s_max[1]), fmaxf(s_max[2], s_max[3]));
    // e is in [-113, 147] for any finite BF16 maximum (2^-133 .. 2^128); 2^-e
    // is then a normal or subnormal float, both exact
    const int e = (m > 0.f) ? 14 - ilogbf(m) : 0;
    if (threadIdx.x == 0) inv_scale[t] = ldexpf(1.0f, -e);
    const int64_t stages = k / kStageK;
    for (int64_t st = threadIdx.x; st < stages; st += blockDim.x) {
        const uint4* src = reinterpret_cast<const uint4*>(row + st * kStageK);
        uint32_t hv[32];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint4 v = src[j];
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const __half lo = __float2half_rn(ldexpf(bf16_lo(w[q]), e));
                const __half hi = __float2half_rn(ldexpf(bf16_hi(w[q]), e));
                hv[4 * j + q] = (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
            }
        }
        uint32_t o[32];
        if (FMT == BQ_T5P8G128 && (st & 1))
            permute_stage<FMT, 1>(hv, o);
        else
            permute_stage<FMT, 0>(hv, o);
        uint4* dst = reinterpret_cast<uint4*>(xh + t * k + st * kStageK);
#pragma unroll
        for (int j = 0; j < 8; ++j) dst[j] = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
    }
}

// ----------------------------------------------------------------- dequant
// The packed bytes and the scale of the 64 weights of one row in one stage.
struct RowChunk {
    uint4 codes;     // binary: 8 bytes; 2-bit: 16 bytes; base-3: 14 bytes from an even offset
    uint32_t scale;  // FP16 bits (0 for rows past the end)
    uint32_t odd;    // base-3: the stage is the second half of its group
};

template <int FMT>
__device__ __forceinline__ RowChunk load_chunk(const Params& p, int64_t row, int64_t st) {
    RowChunk c;
    c.codes = make_uint4(0u, 0u, 0u, 0u);
    c.scale = 0u;
    c.odd = (uint32_t)(st & 1);
    if (row >= p.n) return c;
    const int64_t G = p.k / 128, k0 = st * kStageK;
    c.scale = __ldg(p.scales + row * G + (k0 >> 7));
    if (FMT == BQ_Q1G128) {
        const uint2 b = __ldg(reinterpret_cast<const uint2*>(p.codes + row * (p.k / 8) + (k0 >> 3)));
        c.codes = make_uint4(b.x, b.y, 0u, 0u);
    } else if (FMT == BQ_T2G128) {
        c.codes = __ldg(reinterpret_cast<const uint4*>(p.codes + row * (p.k / 4) + (k0 >> 2)));
    } else {
        // trits 64h .. 64h+63 of the group live in bytes 12h .. 12h+13 (even offset)
        const uint16_t* src =
            reinterpret_cast<const uint16_t*>(p.codes + row * (26 * G) + (k0 >> 7) * 26 + (c.odd ? 12 : 0));
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t lo = __ldg(src + 2 * i);
            const uint32_t hi = (2 * i + 1 < 7) ? (uint32_t)__ldg(src + 2 * i + 1) : 0u;
            w[i] = lo | (hi << 16);
        }
        c.codes = make_uint4(w[0], w[1], w[2], w[3]);
    }
    return c;
}

// Two ternary codes c in {0, 1, 2} held in bits 0-1 and 16-17 -> the FP16
// pair (c - 1) * s.  1024 + c is an exact FP16 (exponent 10, mantissa c);
// subtracting 1025 gives -1, 0 or +1 exactly and the product with s is exact.
__device__ __forceinline__ uint32_t ternary_pair(uint32_t c2, uint32_t ss) {
    uint32_t h;
    asm("{\n\t.reg .b32 v;\n\t"
        "sub.rn.f16x2 v, %1, %2;\n\t"
        "mul.rn.f16x2 %0, v, %3;\n\t}"
        : "=r"(h)
        : "r"(c2 | 0x64006400u), "r"(0x64016401u), "r"(ss));
    return h;
}

// floor(v / 3) of both 16-bit halves (v < 256 each): multiply by 171, shift
// by 9 (exact for v < 256; the low product stays below 2^16, so the halves do
// not interfere once the bits above 7 are masked).
__device__ __forceinline__ uint32_t div3x2(uint32_t v) { return ((v * 171u) >> 9) & 0x007F007Fu; }

// Five base-3 digits of the two bytes in the halves of v -> pairs h[0..4].
// The quotients floor(v / 3^i) come from independent multiply-shifts (171 >> 9,
// 57 >> 9, 19 >> 9, 203 >> 14: exact for every v < 256, and v * m < 2^16, so
// the halves do not interfere once the bits above each quotient are masked),
// and digit i is q_i - 3 q_(i+1); no step waits on the one before.
__device__ __forceinline__ void t5p8_digits(uint32_t v, uint32_t ss, uint32_t* h) {
    const uint32_t q1 = ((v * 171u) >> 9) & 0x007F007Fu, q2 = ((v * 57u) >> 9) & 0x007F007Fu;
    const uint32_t q3 = ((v * 19u) >> 9) & 0x007F007Fu, q4 = ((v * 203u) >> 14) & 0x00030003u;
    h[0] = ternary_pair(v - 3u * q1, ss);
    h[1] = ternary_pair(q1 - 3u * q2, ss);
    h[2] = ternary_pair(q2 - 3u * q3, ss);
    h[3] = ternary_pair(q3 - 3u * q4, ss);
    h[4] = ternary_pair(q4, ss);
}

__device__ __forceinline__ uint32_t byte_of(const uint32_t (&w)[4], int i) { return (w[i >> 2] >> (8 * (i & 3))) & 0xFFu; }

// 64 weights -> 32 FP16 pairs s*q in the kperm order.
template <int FMT>
__device__ __forceinline__ void dequant_chunk(const RowChunk& c, uint32_t (&h)[32]) {
    const uint32_t s = c.scale;
    const uint32_t ss = s | (s << 16);
    const uint32_t w[4] = {c.codes.x, c.codes.y, c.codes.z, c.codes.w};
    if (FMT == BQ_Q1G128) {
        // bit 1 -> +s, bit 0 -> -s: set the FP16 sign where the bit is 0
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const uint32_t nw = ~w[i >> 4];
            const int m = i & 15;
            h[i] = ((nw << (15 - m)) & 0x80008000u) ^ ss;
        }
    } else if (FMT == BQ_T2G128) {
#pragma unroll
        for (int i = 0; i < 32; ++i) h[i] = ternary_pair((w[i >> 3] >> (2 * (i & 7))) & 0x00030003u, ss);
    } else if (!c.odd) {
        // bytes 0..11 paired (j, j+6); byte 12 gives trits 60..63
#pragma unroll
        for (int j = 0; j < 6; ++j) t5p8_digits(byte_of(w, j) | (byte_of(w, j + 6) << 16), ss, h + 5 * j);
        const uint32_t b = byte_of(w, 12) * 0x00010001u;
        const uint32_t x0 = (b & 0xFFFFu) | (div3x2(b) & 0xFFFF0000u);  // (v, v/3)
        const uint32_t x1 = div3x2(x0), x2 = div3x2(x1), x3 = div3x2(x2);
        h[30] = ternary_pair(x0 - 3u * x1, ss);  // digits 0, 1
        h[31] = ternary_pair(x2 - 3u * x3, ss);  // digits 2, 3
    } else {
        // loaded bytes 1..12 paired (j, j+6); byte 0 digit 4 and byte 13 digits 0..2
#pragma unroll
        for (int j = 0; j < 6; ++j) t5p8_digits(byte_of(w, 1 + j) | (byte_of(w, 7 + j) << 16), ss, h + 5 * j);
        const uint32_t y0 = byte_of(w, 0) | (byte_of(w, 13) << 16);
        const uint32_t y1 = div3x2(y0), y2 = div3x2(y1), y3 = div3x2(y2), y4 = div3x2(y3);
        h[30] = ternary_pair((y4 & 0xFFFFu) | ((y0 - 3u * y1) & 0xFFFF0000u), ss);
        h[31] = ternary_pair(((y1 - 3u * y2) >> 16) | ((y2 - 3u * y3) & 0xFFFF0000u), ss);
    }
}

// ----------------------------------------------------------------- units
// Unit u: split fastest, then row tile, then token tile.
struct Unit {
    int64_t mb, nb;
    int split, st_begin, st_end;
};

// (32-bit arithmetic: the host admits only calls with units < 2^31.)
__device__ __forceinline__ Unit unit_of(const Params& p, int64_t mb_count, int spt, int64_t u) {
    Unit w;
    const uint32_t uu = (uint32_t)u, sp = (uint32_t)p.splits, mbc = (uint32_t)mb_count;
    w.split = (int)(uu % sp);
    const uint32_t tile = uu / sp;
    w.mb = tile % mbc;
    w.nb = tile / mbc;
    w.st_begin = (int)((uint32_t)w.split * (uint32_t)spt / sp);
    w.st_end = (int)((uint32_t)(w.split + 1) * (uint32_t)spt / sp);
    return w;
}

// ----------------------------------------------------------------- main
template <int FMT>
__global__ void __launch_bounds__(Roles<FMT>::kThreads, 1) gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_x,
                                                                         const Params p) {
    constexpr int kDequantSets = Roles<FMT>::kSets, kDequantWarps = Roles<FMT>::kDequantWarps;
    constexpr int kTmaWarp = Roles<FMT>::kTmaWarp, kMmaWarp = Roles<FMT>::kMmaWarp;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = ptx::align_smem<1024>(smem_raw);
    uint64_t* full_a = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
    uint64_t* full_b = full_a + kStages;
    uint64_t* empty = full_b + kStages;
    uint64_t* acc_full = empty + kStages;
    uint64_t* acc_empty = acc_full + 2;
    uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(acc_empty + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t mb_count = (p.n + kTileM - 1) / kTileM;
    const int spt = (int)(p.k / kStageK);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            ptx::mbar_init(&full_a[i], kDequantSetWarps);
            ptx::mbar_init(&full_b[i], 1);
            ptx::mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&acc_full[i], 1);
            ptx::mbar_init(&acc_empty[i], kEpiWarps);
        }
        ptx::fence_barrier_init();
    }
    if (warp == kMmaWarp) ptx::tmem_alloc(tmem_base_smem, kTmemCols);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_base_smem;
    ptx::pdl_launch_dependents();
    ptx::pdl_wait();  // X', inv_scale and Y are produced / may be read by earlier kernels

    if (warp < kDequantWarps) {
        // ------------------------------------------------ dequant producers
        const int set = warp / kDequantSetWarps;            // stages it with it % kDequantSets == set
        const int r = (warp % kDequantSetWarps) * 32 + lane;
        int64_t total = 0;  // stages of this CTA
        for (int64_t u = blockIdx.x; u < p.units; u += gridDim.x) {
            const Unit w = unit_of(p, mb_count, spt, u);
            total += w.st_end - w.st_begin;
        }
        // prefetch cursor: unit, its row, next stage
        int64_t pu = blockIdx.x;
        Unit pw = unit_of(p, mb_count, spt, pu);
        int64_t prow = pw.mb * kTileM + r;
        int pst = pw.st_begin;
        auto advance = [&]() {
            if (pu < p.units && ++pst == pw.st_end) {
                pu += gridDim.x;
                if (pu < p.units) {
                    pw = unit_of(p, mb_count, spt, pu);
                    prow = pw.mb * kTileM + r;
                    pst = pw.st_begin;
                }
            }
        };
        // this set's next stage: load it, then step over the other sets' stages
        auto next_chunk = [&]() {
            RowChunk c = {make_uint4(0u, 0u, 0u, 0u), 0u, 0u};
            if (pu < p.units) c = load_chunk<FMT>(p, prow, pst);
#pragma unroll
            for (int i = 0; i < kDequantSets; ++i) advance();
            return c;
        };
        for (int i = 0; i < set; ++i) advance();
        const int64_t mine = (total - set + kDequantSets - 1) / kDequantSets;  // stages of this set
        RowChunk pipe[kAhead];
#pragma unroll
        for (int i = 0; i < kAhead; ++i) pipe[i] = next_chunk();
        bool alive = true;
        if constexpr (FMT == BQ_T5P8G128) {
            // the base-3 decode is long: one copy of it in a loop that shifts
            // the ring of chunks by one entry per stage (the unrolled form below
            // keeps kAhead copies; for this format the instruction fetch of
            // those copies measurably stalled the dequant warps)
#pragma unroll 1
            for (int64_t j = 0; j < mine; ++j) {
                const int64_t it = j * kDequantSets + set;  // stage index of the CTA's sequence
                const int slot = (int)(it % kStages);
                if (it >= kStages &&
                    !ptx::mbar_wait_bounded(&empty[slot], (uint32_t)(((it / kStages) - 1) & 1), kWaitPolls)) {
                    record_status(p.status, BQ_ERR_TIMEOUT);
                    break;
                }
                uint32_t h[32];
                dequant_chunk<FMT>(pipe[0], h);
#pragma unroll
                for (int i = 0; i + 1 < kAhead; ++i) pipe[i] = pipe[i + 1];
                pipe[kAhead - 1] = next_chunk();
                uint8_t* a = smem + slot * kStageBytes + r * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<uint4*>(a + ((c ^ (r & 7)) << 4)) =
                        make_uint4(h[4 * c], h[4 * c + 1], h[4 * c + 2], h[4 * c + 3]);
                ptx::fence_proxy_async_smem();  // generic-proxy stores -> visible to the tensor core
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&full_a[slot]);
            }
            alive = false;  // (the loop below is for the other formats)
        }
        // unrolled by kAhead so that each ring entry is a fixed set of registers:
        // a chunk is consumed kAhead stages after its load was issued
        for (int64_t base = 0; base < mine && alive; base += kAhead) {
#pragma unroll
            for (int i = 0; i < kAhead; ++i) {
                const int64_t it = (base + i) * kDequantSets + set;  // stage index of the CTA's sequence
                if (base + i < mine && alive) {
                    const int slot = (int)(it % kStages);
                    if (it >= kStages &&
                        !ptx::mbar_wait_bounded(&empty[slot], (uint32_t)(((it / kStages) - 1) & 1), kWaitPolls)) {
                        record_status(p.status, BQ_ERR_TIMEOUT);
                        alive = false;
                    } else {
                        uint32_t h[32];
                        dequant_chunk<FMT>(pipe[i], h);
                        pipe[i] = next_chunk();
                        uint8_t* a = smem + slot * kStageBytes + r * 128;
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            *reinterpret_cast<uint4*>(a + ((c ^ (r & 7)) << 4)) =
                                make_uint4(h[4 * c], h[4 * c + 1], h[4 * c + 2], h[4 * c + 3]);
                        ptx::fence_proxy_async_smem();  // generic-proxy stores -> visible to the tensor core
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive(&full_a[slot]);
                    }
                }
            }
        }
    } else if (warp == kTmaWarp) {
        // ------------------------------------------------ activation TMA
        if (lane == 0) {
            ptx::prefetch_tensormap(&tm_x);
            const uint32_t bytes = (uint32_t)p.tile_n * kStageK * 2;
            int64_t it = 0;
            bool alive = true;
            for (int64_t u = blockIdx.x; u < p.units && alive; u += gridDim.x) {
                const Unit w = unit_of(p, mb_count, spt, u);
                for (int st = w.st_begin; st < w.st_end; ++st, ++it) {
                    const int slot = (int)(it % kStages);
                    if (it >= kStages &&
                        !ptx::mbar_wait_bounded(&empty[slot], (uint32_t)(((it / kStages) - 1) & 1), kWaitPolls)) {
                        record_status(p.status, BQ_ERR_TIMEOUT);
                        alive = false;
                        break;
                    }
                    ptx::mbar_arrive_expect_tx(&full_b[slot], bytes);
                    ptx::tma_load_2d(smem + slot * kStageBytes + kABytes, &tm_x, st * kStageK,
                                     (int32_t)(w.nb * p.tile_n), &full_b[slot]);
                }
            }
            // the last copies must land before this CTA may exit
            const int64_t issued = it;
            for (int64_t j = (issued > kStages ? issued - kStages : 0); j < issued; ++j)
                if (!ptx::mbar_wait_bounded(&full_b[j % kStages], (uint32_t)((j / kStages) & 1), kWaitPolls))
                    record_status(p.status, BQ_ERR_TIMEOUT);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            // D f32, A f16, B f16, both K-major, N = tile_n, M = 128
            const uint32_t idesc = (1u << 4) | ((uint32_t)(p.tile_n >> 3) << 17) | (8u << 24);
            int64_t it = 0, local = 0;
            bool ok = true;
            for (int64_t u = blockIdx.x; u < p.units && ok; u += gridDim.x, ++local) {
                const Unit w = unit_of(p, mb_count, spt, u);
                const int ab = (int)(local & 1);
                if (local >= 2 &&
                    !ptx::mbar_wait_bounded(&acc_empty[ab], (uint32_t)(((local >> 1) - 1) & 1), kWaitPolls)) {
                    record_status(p.status, BQ_ERR_TIMEOUT);
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                for (int st = w.st_begin; st < w.st_end; ++st, ++it) {
                    const int slot = (int)(it % kStages);
                    const uint32_t par = (uint32_t)((it / kStages) & 1);
                    if (!ptx::mbar_wait_bounded(&full_a[slot], par, kWaitPolls) ||
                        !ptx::mbar_wait_bounded(&full_b[slot], par, kWaitPolls)) {
                        record_status(p.status, BQ_ERR_TIMEOUT);
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t a0 = ptx::smem_u32(smem + slot * kStageBytes);
                    const uint32_t b0 = a0 + kABytes;
#pragma unroll
                    for (int kk = 0; kk < kStageK / 16; ++kk) {
                        const uint64_t ad = ptx::smem_desc_kmajor_sw128(a0 + kk * 32);
                        const uint64_t bd = ptx::smem_desc_kmajor_sw128(b0 + kk * 32);
                        ptx::mma_f16_ss(tmem + ab * kMaxTileN, ad, bd, idesc, (st > w.st_begin || kk > 0) ? 1u : 0u);
                    }
                    ptx::tc_commit(&empty[slot]);
                }
                if (ok) ptx::tc_commit(&acc_full[ab]);
            }
        }
    } else {
        // ------------------------------------------------ epilogue
        const int quad = warp & 3;  // TMEM lane quadrant this warp may access
        const int r = quad * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
        int64_t local = 0;
        for (int64_t u = blockIdx.x; u < p.units; u += gridDim.x, ++local) {
            const Unit w = unit_of(p, mb_count, spt, u);
            const int ab = (int)(local & 1);
            if (!ptx::mbar_wait_bounded(&acc_full[ab], (uint32_t)((local >> 1) & 1), kWaitPolls)) {
                record_status(p.status, BQ_ERR_TIMEOUT);
                break;
            }
            ptx::tc_fence_after();
            const int64_t row = w.mb * kTileM + r;
            float* part = p.partial + (int64_t)w.split * p.t * p.n;
#pragma unroll 1
            for (int c0 = 0; c0 < p.tile_n; c0 += 32) {
                uint32_t v[32];
                ptx::tmem_ld_x32(tmem + lane_base + ab * kMaxTileN + c0, v);
                ptx::tc_wait_ld();
                const int64_t t0 = w.nb * p.tile_n + c0;
                if (row < p.n) {
                    if (p.splits == 1) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int64_t tok = t0 + j;
                            if (tok < p.t) {
                                const float yv = __uint_as_float(v[j]) * __ldg(p.inv_scale + tok);
                                if (p.y_f32)
                                    static_cast<float*>(p.y)[tok * p.n + row] = yv;
                                else
                                    static_cast<uint16_t*>(p.y)[tok * p.n + row] = float_to_bf16_bits(yv);
                            }
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int64_t tok = t0 + j;
                            if (tok < p.t) part[tok * p.n + row] = __uint_as_float(v[j]);
                        }
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&acc_empty[ab]);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

// Sum of the split partial tiles in split order, times 2^-e_t, as BF16 or FP32.
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float* __restrict__ partial, int splits,
                                                            const float* __restrict__ inv_scale, void* __restrict__ y,
                                                            int y_f32, int64_t t, int64_t n) {
    ptx::pdl_wait();
    const int64_t total = t * n;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        float acc = 0.0f;
        for (int s = 0; s < splits; ++s) acc += partial[s * total + i];
        const float yv = acc * inv_scale[i / n];
        if (y_f32)
            static_cast<float*>(y)[i] = yv;
        else
            static_cast<uint16_t*>(y)[i] = float_to_bf16_bits(yv);
    }
}

// ----------------------------------------------------------------- host

// Tile shape, K split and grid of one call.
struct Plan {
    int tile_n, splits;
    int64_t units, grid;
};

Plan plan_of(int64_t n, int64_t k, int64_t t) {
    Plan pl;
    const int64_t nb = (t + kMaxTileN - 1) / kMaxTileN;
    const int64_t per = (t + nb - 1) / nb;
    pl.tile_n = (int)((per + 31) / 32 * 32);
    const int64_t tiles = ((n + kTileM - 1) / kTileM) * nb;
    const int64_t sms = sm_count(), spt = k / kStageK;
    int64_t splits = 1;
    if (tiles < sms) {
        splits = sms / tiles;
        const int64_t cap = spt / 4 > 1 ? spt / 4 : 1;  // at least 4 stages per split
        if (splits > cap) splits = cap;
        if (splits < 1) splits = 1;
    }
    pl.splits = (int)splits;
    pl.units = tiles * splits;
    pl.grid = pl.units < sms ? pl.units : sms;
    return pl;
}

inline int64_t align256(int64_t b) { return (b + 255) / 256 * 256; }

template <int FMT>
cudaError_t launch_typed(Params prm, const Plan& pl, const uint16_t* x, uint16_t* xh, float* inv_scale, cudaStream_t s) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    {
        const cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(gemm_tc_kernel<FMT>), kSmemBytes);
        if (e != cudaSuccess) return e;
    }
    CUtensorMap tm_x;
    {
        cuuint64_t dims[2] = {(cuuint64_t)prm.k, (cuuint64_t)prm.t};
        cuuint64_t strides[1] = {(cuuint64_t)(prm.k * 2)};
        cuuint32_t box[2] = {(cuuint32_t)kStageK, (cuuint32_t)pl.tile_n};
        cuuint32_t es[2] = {1, 1};
        if (enc(&tm_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, xh, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)prm.t);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, xprep_f16_kernel<FMT>, x, (int64_t)prm.k, xh, inv_scale);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3((unsigned)pl.grid);
    cfg.blockDim = dim3(Roles<FMT>::kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    e = cudaLaunchKernelEx(&cfg, gemm_tc_kernel<FMT>, tm_x, prm);
    if (e != cudaSuccess) return e;
    if (pl.splits > 1) {
        const int64_t total = prm.t * prm.n;
        int64_t blocks = (total + 255) / 256;
        const int64_t cap = 8 * (int64_t)sm_count();
        cfg.gridDim = dim3((unsigned)(blocks < cap ? blocks : cap));
        cfg.blockDim = dim3(256);
        cfg.dynamicSmemBytes = 0;
        e = cudaLaunchKernelEx(&cfg, splitk_reduce_kernel, (const float*)prm.partial, pl.splits,
                               (const float*)inv_scale, prm.y, prm.y_f32, prm.t, prm.n);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

}  // namespace gemm

// Workspace of the tensor-core GEMM: FP16 activations [T][K], inverse
// pre-scales [T] and, when K is split, the FP32 partial tiles
// [splits][T][N] (256-byte aligned pieces).
int64_t gemm_tc_workspace_bytes(int64_t n, int64_t k, int64_t t) {
    const gemm::Plan pl = gemm::plan_of(n, k, t);
    int64_t b = gemm::align256(t * k * 2) + gemm::align256(t * 4);
    if (pl.splits > 1) b += gemm::align256((int64_t)pl.splits * t * n * 4);
    return b;
}

// Kernels one call launches: activation prep, GEMM, and the split-K reduction
// when K is split.
int gemm_tc_launches(int64_t n, int64_t k, int64_t t) { return gemm::plan_of(n, k, t).splits > 1 ? 3 : 2; }

bool gemm_tc_eligible(int fmt, int64_t n, int64_t k, int64_t t) {
    if (!((fmt == BQ_Q1G128 || fmt == BQ_T2G128 || fmt == BQ_T5P8G128) && n > 0 && k > 0 && k % 128 == 0 &&
          t > 0 && t <= (int64_t)INT32_MAX && n <= (int64_t)INT32_MAX && k / 64 <= (int64_t)(1 << 22)))
        return false;
    return gemm::plan_of(n, k, t).units < ((int64_t)1 << 31);
}

cudaError_t launch_gemm_tc(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                           const uint16_t* x, int64_t t, void* y, int y_dtype, void* workspace, cudaStream_t s) {
    const gemm::Plan pl = gemm::plan_of(n, k, t);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint16_t* xh = reinterpret_cast<uint16_t*>(ws);
    float* inv = reinterpret_cast<float*>(ws + gemm::align256(t * k * 2));
    float* part = reinterpret_cast<float*>(ws + gemm::align256(t * k * 2) + gemm::align256(t * 4));
    gemm::Params prm;
    prm.codes = codes;
    prm.scales = scales;
    prm.inv_scale = inv;
    prm.y = y;
    prm.y_f32 = y_dtype == BQ_F32 ? 1 : 0;
    prm.partial = pl.splits > 1 ? part : nullptr;
    prm.n = n;
    prm.k = k;
    prm.t = t;
    prm.units = pl.units;
    prm.tile_n = pl.tile_n;
    prm.splits = pl.splits;
    prm.status = device_status_ptr();
    if (!prm.status) return cudaErrorUnknown;
    if (fmt == BQ_Q1G128) return gemm::launch_typed<BQ_Q1G128>(prm, pl, x, xh, inv, s);
    if (fmt == BQ_T2G128) return gemm::launch_typed<BQ_T2G128>(prm, pl, x, xh, inv, s);
    return gemm::launch_typed<BQ_T5P8G128>(prm, pl, x, xh, inv, s);
}

}  // namespace bq
