// Weight-streaming GEMV with tensor-core accumulation of the decoded codes
// (binary g128 and 2-bit-slot ternary g128, batch 1..4, K % 1024 == 0).
//
// Why the tensor core: at batch 1 the binary format must be consumed at
// ~126 weights per clock per SM to stream HBM at 80% of its bandwidth, while
// the integer/logic pipe retires 64 operations per clock per SM; any CUDA-core
// decode that spends half an operation per weight cannot get there (the
// "1-bit Bonsai 8B" notes, section 4.4, observe the same shift of inline
// dequantisation towards compute).  So the codes are expanded with a handful of
// LOP3s into int8 operands and the multiply-accumulate runs on the tensor core.
//
// Why the register-fed warp MMA (mma.sync) rather than tcgen05: with N = 8
// activation columns the tcgen05 MMA (M = 128, K = 32, int8) has a floor of
// ~46-56 cycles per instruction whatever N is (measured on B200), i.e. at most
// ~89 A-operand bytes per clock per SM, below the 126 needed; the warp MMA
// m16n8k32 retires 256 A bytes per clock per SM.  tcgen05 is used where the
// contraction is dense (the prefill GEMM).
//
//   binary  : byte j of (w & (0x01010101 << p)) is 2^p * bit(8j+p) of the code
//             word w -- eight masks turn one 32-bit word into eight operand
//             registers with no shift.  The activation operand of that k-slot
//             carries Q_k / 2^p, so the product is bit * Q_k exactly.
//   2-bit   : byte j of (w & (0x03030303 << 2i)) is 4^i * c, c = q+1 the code
//             of trit 4j+i -- four masks per word, again no shift; the
//             activation operand of that k-slot carries Q_k / 4^i.
//
// Q_k is the activation in fixed point: per (batch row b, group g) a power of
// two 2^E maps the group's largest |x| into [2^29, 2^30); Q = round(x 2^E)
// (rounded to a multiple of 2^7, binary, or 2^6, 2-bit, so that Q / 2^p and
// Q / 4^i stay integers).
// Q is split into four signed base-256 digits, one MMA column each, and the
// int32 column sums are recombined in FP32.  Per group and row:
//   binary : y += s * (2 * 2^-E * sum_k bit_k Q_k - 2^-E * sum_k Q_k)
//   ternary: y += s * (    2^-E * sum_k c_k   Q_k - 2^-E * sum_k Q_k)
// (sum of s * q * x with q = 2 bit - 1, resp. q = c - 1; "Bonsai-27B ...
// Binary g128" section on the representation: 0 -> -scale, 1 -> +scale).  The
// only rounding before the FP32 recombination is that of x to Q: at most
// 2^6 units of 2^-E per element, i.e. 2^-23 of the group's largest |x|.
//
// Data movement: per pipeline stage (1024 weights of K for 128 rows) a
// producer warp issues a TMA tile load of the codes (128-byte swizzle), one of
// the FP16 scales and a bulk copy of the prepared activation operands into
// shared memory; eight compute warps read conflict-free from there.  The grid
// is persistent (two CTAs per SM) and splits the sequence of (row block,
// stage) items evenly ("stream-K"), so there is no tail wave; a row block
// shared by two CTAs is finished by the last of them, which adds the partial
// sums in CTA order (deterministic).  Launches use programmatic dependent
// launch: a call's weight stream starts while the previous kernel in the
// stream is still draining.
#include <cuda.h>

#include "bq_internal.cuh"
#include "bq_ptx.cuh"

namespace bq {
namespace tc {

constexpr int kGroupsPerStage = 8;
constexpr int kRowsPerCta = 128;
constexpr int kComputeWarps = 8;
constexpr int kRowTiles = 1;  // 16-row MMA tiles per compute warp
constexpr int kThreads = (kComputeWarps + 1) * 32;
constexpr int kBfragBytesPerGroup = 4 * 32 * 8;  // 4 MMAs x 32 lanes x (b0, b1)
constexpr int kTableBytesPerGroup = 4 * 16;      // 4 lanes-in-quad x float4
constexpr int kXTileBytes = kGroupsPerStage * (kBfragBytesPerGroup + kTableBytesPerGroup);  // 8704
constexpr uint32_t kWaitPolls = 1u << 23;

template <int FMT>
struct Fmt;
template <>
struct Fmt<BQ_Q1G128> {
    static constexpr int kRowBytesPerStage = 128;  // 8 groups x 16 bytes
    static constexpr int kCoefShift = 1;           // y uses 2 * sum(bit * x) - sum(x)
};
template <>
struct Fmt<BQ_T2G128> {
    static constexpr int kRowBytesPerStage = 256;  // 8 groups x 32 bytes
    static constexpr int kCoefShift = 0;           // y uses sum(c * x) - sum(x)
};

template <int FMT, int NT>
struct Layout {
    static constexpr int kCodesBytes = kRowsPerCta * Fmt<FMT>::kRowBytesPerStage;
    static constexpr int kScalesBytes = kRowsPerCta * kGroupsPerStage * 2;
    static constexpr int kXBytes = NT * kXTileBytes;
    static constexpr int kStageBytes = (kCodesBytes + kScalesBytes + kXBytes + 1023) / 1024 * 1024;
    // two CTAs per SM: 4 (binary, batch <= 2), 3 (binary, batch <= 4) or 2 (2-bit) stages
    static constexpr int kStages = (FMT == BQ_Q1G128) ? (NT == 1 ? 4 : 3) : 2;
    static_assert(kComputeWarps * 16 * kRowTiles == kRowsPerCta, "row tiling");
    static constexpr int kSmemBytes = kStages * kStageBytes + 1024 + 2 * kStages * 8;
};

struct Params {
    const uint8_t* xdata;     // prepared activation operands, [stage][NT][kXTileBytes]
    float* partial;           // [grid][2][batch][kRowsPerCta] partial sums of split row blocks
    unsigned int* counters;   // [row_blocks], zeroed by the prep kernel
    void* y;
    int y_dtype;
    int batch;
    int64_t n;
    int stages_total;
    int row_blocks;
    int* status;
};

__device__ __forceinline__ void named_barrier_compute() {
    asm volatile("bar.sync 1, %0;" ::"n"(kComputeWarps * 32) : "memory");
}

// ----------------------------------------------------------------- prep
// One CTA per stage (8 groups).  Writes, for each n-tile (two batch rows x four
// digits), the B fragments of the 32 MMAs of the stage in lane order and the
// per-(group, lane-in-quad) recombination table {2^a, 2^b, sum term, 0}.
template <int FMT, int NT>
__global__ void __launch_bounds__(256) prep_kernel(const uint16_t* __restrict__ x, int64_t k, int batch,
                                                   uint8_t* __restrict__ xdata, unsigned int* counters,
                                                   int row_blocks) {
    __shared__ int8_t dig[2 * NT][kGroupsPerStage * 128][4];
    const int st = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Let the GEMV kernel launch and prefetch weights now; x and the workspace
    // are touched only after the previous kernel in the stream has finished.
    ptx::pdl_launch_dependents();
    ptx::pdl_wait();
    if (st == 0)
        for (int i = threadIdx.x; i < row_blocks; i += blockDim.x) counters[i] = 0u;
    uint8_t* out = xdata + (size_t)st * NT * kXTileBytes;

    const int G = warp;  // 8 warps <-> 8 groups of the stage
    const int64_t kbase = ((int64_t)st * kGroupsPerStage + G) * 128;
    // Per n-tile: does any batch row of this group need the two-factor
    // recombination (2^e below the normal FP32 range)?  The flag is shared by
    // the group's four table entries so that the GEMV kernel's choice is
    // uniform across the warp.
    bool two_factor[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) two_factor[nt] = false;
    for (int bb = 0; bb < 2 * NT && bb < batch; ++bb) {
        const uint2 raw = *reinterpret_cast<const uint2*>(x + bb * k + kbase + lane * 4);
        float m = fmaxf(fmaxf(fabsf(bf16_lo(raw.x)), fabsf(bf16_hi(raw.x))),
                        fmaxf(fabsf(bf16_lo(raw.y)), fabsf(bf16_hi(raw.y))));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        const int E = (m > 0.f) ? 29 - ilogbf(m) : 0;
        if (Fmt<FMT>::kCoefShift - E < -126) two_factor[bb >> 1] = true;
    }
    for (int bb = 0; bb < 2 * NT; ++bb) {
        float xv[4] = {0.f, 0.f, 0.f, 0.f};
        if (bb < batch) {
            const uint2 raw = *reinterpret_cast<const uint2*>(x + bb * k + kbase + lane * 4);
            xv[0] = bf16_lo(raw.x); xv[1] = bf16_hi(raw.x); xv[2] = bf16_lo(raw.y); xv[3] = bf16_hi(raw.y);
        }
        float m = fmaxf(fmaxf(fabsf(xv[0]), fabsf(xv[1])), fmaxf(fabsf(xv[2]), fabsf(xv[3])));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        const int E = (m > 0.f) ? 29 - ilogbf(m) : 0;
        long long sumq = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int kk = lane * 4 + i;  // position in the group
            int q, b;
            if (FMT == BQ_Q1G128) {
                q = __float2int_rn(ldexpf(xv[i], E - 7)) * 128;
                b = q >> (kk & 7);  // exact: q is a multiple of 2^7
            } else {
                q = __float2int_rn(ldexpf(xv[i], E - 6)) * 64;
                b = q >> (2 * (kk & 3));  // exact: q is a multiple of 2^6
            }
            sumq += q;
            const int d0 = (int8_t)(b & 0xFF);
            b = (b - d0) >> 8;
            const int d1 = (int8_t)(b & 0xFF);
            b = (b - d1) >> 8;
            const int d2 = (int8_t)(b & 0xFF);
            const int d3 = (b - d2) >> 8;
            int8_t* dst = dig[bb][G * 128 + kk];
            dst[0] = (int8_t)d0; dst[1] = (int8_t)d1; dst[2] = (int8_t)d2; dst[3] = (int8_t)d3;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sumq += __shfl_xor_sync(0xffffffffu, sumq, off);
        if (lane < 2) {
            const int h = lane;  // digit pair (0,1) or (2,3)
            const int t = 2 * (bb & 1) + h;
            const int nt = bb >> 1;
            const int e = Fmt<FMT>::kCoefShift - E + 16 * h;
            // one factor 2^e when it is a normal float, else 2^a * 2^(e-a)
            const bool two = two_factor[nt];
            const int a = two ? max(-60, min(60, e)) : e;
            float4 tab;
            tab.x = ldexpf(1.0f, a);
            tab.y = ldexpf(1.0f, e - a);
            tab.z = (h == 0) ? (float)ldexp((double)sumq, -E) : 0.0f;
            tab.w = two ? 1.0f : 0.0f;
            *reinterpret_cast<float4*>(out + nt * kXTileBytes + kGroupsPerStage * kBfragBytesPerGroup +
                                       (G * 4 + t) * 16) = tab;
        }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < NT * kGroupsPerStage * 4 * 32; idx += blockDim.x) {
        const int ln = idx & 31, q = (idx >> 5) & 3, g8 = (idx >> 7) & 7, nt = idx >> 10;
        const int gq = ln >> 2, t = ln & 3;
        const int bb = nt * 2 + (gq >> 2), dg = gq & 3;
        uint32_t b0 = 0, b1 = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int k0, k1;
            if (FMT == BQ_Q1G128) {
                k0 = 32 * t + 8 * j + 2 * q;
                k1 = k0 + 1;
            } else {
                k0 = 32 * t + 4 * j + q;  // word 2t of the row's group, class q
                k1 = k0 + 16;             // word 2t+1
            }
            b0 |= (uint32_t)(uint8_t)dig[bb][g8 * 128 + k0][dg] << (8 * j);
            b1 |= (uint32_t)(uint8_t)dig[bb][g8 * 128 + k1][dg] << (8 * j);
        }
        // lane-contiguous 16 bytes hold (b0, b1) of MMAs 2j and 2j+1 of the group
        *reinterpret_cast<uint2*>(out + nt * kXTileBytes + ((g8 * 2 + (q >> 1)) * 32 + ln) * 16 + (q & 1) * 8) =
            make_uint2(b0, b1);
    }
}

// ----------------------------------------------------------------- main
// Persistent stream-K kernel.  The work is the sequence of items
// (row block, stage) in row-block-major order; CTA c takes items
// [c*T/C, (c+1)*T/C).  A row block whose stages all fall inside one CTA is
// written directly; a row block split between CTAs is combined by the CTA that
// finishes it last, adding the partial sums in CTA order (deterministic).
__host__ __device__ __forceinline__ int64_t item_begin(int64_t c, int64_t T, int64_t C) { return c * T / C; }
__device__ __forceinline__ int64_t cta_of_item(int64_t i, int64_t T, int64_t C) { return ((i + 1) * C - 1) / T; }

template <int FMT, int NT>
__global__ void __launch_bounds__(kThreads, 2) gemv_tc_kernel(const __grid_constant__ CUtensorMap tm_codes,
                                                              const __grid_constant__ CUtensorMap tm_scales,
                                                              const Params p) {
    using L = Layout<FMT, NT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = ptx::align_smem<1024>(smem_raw);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kStages * L::kStageBytes);
    uint64_t* empty = full + L::kStages;
    __shared__ int s_last;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t S = p.stages_total, T = (int64_t)p.row_blocks * S, C = gridDim.x, c = blockIdx.x;
    const int64_t it0 = item_begin(c, T, C), it1 = item_begin(c + 1, T, C);
    const int nit = (int)(it1 - it0);

    if (threadIdx.x == 0) {
        for (int i = 0; i < L::kStages; ++i) {
            ptx::mbar_init(&full[i], 1);
            ptx::mbar_init(&empty[i], kComputeWarps);
        }
        ptx::fence_barrier_init();
    }
    __syncthreads();
    // The next grid in the stream may start its prologue (and its own weight
    // prefetch) as soon as SMs free up; it waits for this grid before it reads
    // anything this grid writes.
    ptx::pdl_launch_dependents();

    if (warp == kComputeWarps) {
        // ------------------------------------------------ producer
        if (lane == 0) {
            ptx::prefetch_tensormap(&tm_codes);
            ptx::prefetch_tensormap(&tm_scales);
            // (row block, stage) of the next weight tile and stage of the next
            // activation tile, advanced without divisions
            int w_rb = (int)(it0 / S), w_st = (int)(it0 % S), x_st = w_st;
            auto issue_weights = [&](int it) {
                const int slot = it % L::kStages;
                uint8_t* sb = smem + slot * L::kStageBytes;
                const int rb = w_rb, st = w_st;
                if (++w_st == (int)S) {
                    w_st = 0;
                    ++w_rb;
                }
                ptx::mbar_arrive_expect_tx(&full[slot], L::kCodesBytes + L::kScalesBytes + L::kXBytes);
#pragma unroll
                for (int box = 0; box < Fmt<FMT>::kRowBytesPerStage / 128; ++box)
                    ptx::tma_load_2d(sb + box * (kRowsPerCta * 128), &tm_codes,
                                     st * Fmt<FMT>::kRowBytesPerStage + box * 128, rb * kRowsPerCta, &full[slot]);
                ptx::tma_load_2d(sb + L::kCodesBytes, &tm_scales, st * kGroupsPerStage, rb * kRowsPerCta,
                                 &full[slot]);
            };
            auto issue_x = [&](int it) {
                const int slot = it % L::kStages;
                uint8_t* sb = smem + slot * L::kStageBytes;
                const int st = x_st;
                if (++x_st == (int)S) x_st = 0;
                ptx::bulk_load(sb + L::kCodesBytes + L::kScalesBytes, p.xdata + (size_t)st * L::kXBytes,
                               L::kXBytes, &full[slot]);
            };
            // The weights do not depend on the previous kernel: start streaming
            // them before waiting for it; the activation operands come after.
            const int pre = nit < L::kStages ? nit : L::kStages;
            for (int it = 0; it < pre; ++it) issue_weights(it);
            ptx::pdl_wait();
            for (int it = 0; it < pre; ++it) issue_x(it);
            int issued = pre;
            for (int it = pre; it < nit; ++it) {
                const int slot = it % L::kStages;
                if (!ptx::mbar_wait_bounded(&empty[slot], ((it / L::kStages) - 1) & 1, kWaitPolls)) {
                    record_status(p.status, BQ_ERR_TIMEOUT);
                    break;
                }
                issue_weights(it);
                issue_x(it);
                issued = it + 1;
            }
            // every copy this CTA issued must land before it may exit
            for (int it = (issued > L::kStages ? issued - L::kStages : 0); it < issued; ++it)
                if (!ptx::mbar_wait_bounded(&full[it % L::kStages], (it / L::kStages) & 1, kWaitPolls))
                    record_status(p.status, BQ_ERR_TIMEOUT);
        }
        return;
    }

    // ---------------------------------------------------- compute warps
    const int g = lane >> 2, t = lane & 3;
    const bool writer = (t & 1) == 0;
    float yacc[kRowTiles][NT][2];
#pragma unroll
    for (int j = 0; j < kRowTiles; ++j)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) yacc[j][nt][0] = yacc[j][nt][1] = 0.0f;

    bool alive = true;
    // (row block, stage) of the current item, advanced without divisions
    int rb = (int)(it0 / S), st = (int)(it0 % S);
    const int Si = (int)S;
    // lanes whose B-fragment columns hold batch rows that exist (at batch 1 the
    // upper four columns are zero and are not read)
    const bool b_live = g < 4 * (p.batch < 2 ? p.batch : 2);
    for (int it = 0; it < nit; ++it, (++st == Si) ? (st = 0, ++rb) : 0) {
        const int slot = it % L::kStages;
        if (alive && !ptx::mbar_wait_bounded(&full[slot], (it / L::kStages) & 1, kWaitPolls)) {
            record_status(p.status, BQ_ERR_TIMEOUT);
            alive = false;
        }
        if (alive) {
            const uint8_t* stage = smem + slot * L::kStageBytes;
            const uint8_t* codes_s = stage;
            const uint16_t* scales_s = reinterpret_cast<const uint16_t*>(stage + L::kCodesBytes);
            const uint8_t* x_s = stage + L::kCodesBytes + L::kScalesBytes;
            const int r0 = warp * 16 + g;  // this thread's rows: r0 and r0 + 8
            // the 8 group scales of both rows (FP16 pairs)
            const uint4 sv0 = *reinterpret_cast<const uint4*>(scales_s + r0 * kGroupsPerStage);
            const uint4 sv1 = *reinterpret_cast<const uint4*>(scales_s + (r0 + 8) * kGroupsPerStage);
            const uint32_t s0w[4] = {sv0.x, sv0.y, sv0.z, sv0.w};
            const uint32_t s1w[4] = {sv1.x, sv1.y, sv1.z, sv1.w};
#pragma unroll
            for (int G = 0; G < kGroupsPerStage; ++G) {
                uint4 bf[NT][2];
                float4 tab[NT];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const uint8_t* xt = x_s + nt * kXTileBytes;
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        bf[nt][h] = (nt > 0 || b_live)
                                        ? *reinterpret_cast<const uint4*>(xt + ((G * 2 + h) * 32 + lane) * 16)
                                        : make_uint4(0u, 0u, 0u, 0u);
                    tab[nt] = *reinterpret_cast<const float4*>(xt + kGroupsPerStage * kBfragBytesPerGroup + (G * 4 + t) * 16);
                }
                int acc[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0;
                if (FMT == BQ_Q1G128) {
                    const int off = ((G ^ g) << 4) + 4 * t;
                    const uint32_t w0 = *reinterpret_cast<const uint32_t*>(codes_s + r0 * 128 + off);
                    const uint32_t w1 = *reinterpret_cast<const uint32_t*>(codes_s + (r0 + 8) * 128 + off);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t m0 = 0x01010101u << (2 * q), m1 = 0x01010101u << (2 * q + 1);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const uint32_t b0 = (q & 1) ? bf[nt][q >> 1].z : bf[nt][q >> 1].x;
                            const uint32_t b1 = (q & 1) ? bf[nt][q >> 1].w : bf[nt][q >> 1].y;
                            ptx::mma_u8s8(acc[nt], w0 & m0, w1 & m0, w0 & m1, w1 & m1, b0, b1);
                        }
                    }
                } else {
                    // words 2t, 2t+1 of the row's 32-byte group: one 8-byte load per row
                    const uint8_t* box = codes_s + (G >> 2) * (kRowsPerCta * 128);
                    const int chunk = 2 * (G & 3) + (t >> 1);
                    const int off = ((chunk ^ g) << 4) + 8 * (t & 1);
                    const uint2 wr0 = *reinterpret_cast<const uint2*>(box + r0 * 128 + off);
                    const uint2 wr1 = *reinterpret_cast<const uint2*>(box + (r0 + 8) * 128 + off);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t m = 0x03030303u << (2 * q);
                        const uint32_t a0 = wr0.x & m, a1 = wr1.x & m, a2 = wr0.y & m, a3 = wr1.y & m;
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const uint32_t b0 = (q & 1) ? bf[nt][q >> 1].z : bf[nt][q >> 1].x;
                            const uint32_t b1 = (q & 1) ? bf[nt][q >> 1].w : bf[nt][q >> 1].y;
                            ptx::mma_u8s8(acc[nt], a0, a1, a2, a3, b0, b1);
                        }
                    }
                }
                const float s0 = half_bits_to_float((uint16_t)(s0w[G >> 1] >> (16 * (G & 1))));
                const float s1 = half_bits_to_float((uint16_t)(s1w[G >> 1] >> (16 * (G & 1))));
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    // D0 + 256 D1 is exact in int32 (|D| < 2^21)
                    const float v0 = (float)(acc[nt][0] + 256 * acc[nt][1]);
                    const float v1 = (float)(acc[nt][2] + 256 * acc[nt][3]);
                    float u0, u1;
                    if (tab[nt].w == 0.0f) {  // uniform across the warp (one group)
                        u0 = fmaf(v0, tab[nt].x, -tab[nt].z);
                        u1 = fmaf(v1, tab[nt].x, -tab[nt].z);
                    } else {
                        u0 = fmaf(v0 * tab[nt].x, tab[nt].y, -tab[nt].z);
                        u1 = fmaf(v1 * tab[nt].x, tab[nt].y, -tab[nt].z);
                    }
                    yacc[0][nt][0] = fmaf(s0, u0, yacc[0][nt][0]);
                    yacc[0][nt][1] = fmaf(s1, u1, yacc[0][nt][1]);
                }
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&empty[slot]);
        }
        // ---------------------------------------- row block finished here?
        if (st != S - 1 && it != nit - 1) continue;
#pragma unroll
        for (int j = 0; j < kRowTiles; ++j)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int r = 0; r < 2; ++r) yacc[j][nt][r] += __shfl_xor_sync(0xffffffffu, yacc[j][nt][r], 1);
        const int64_t rb_first = (int64_t)rb * S, rb_last = rb_first + S - 1;
        const bool whole = rb_first >= it0 && rb_last < it1;
        if (whole) {
            if (writer) {
#pragma unroll
                for (int j = 0; j < kRowTiles; ++j)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int r = 0; r < 2; ++r) {
                            const int bb = nt * 2 + (t >> 1);
                            const int64_t row = (int64_t)rb * kRowsPerCta + warp * (16 * kRowTiles) + j * 16 + g + 8 * r;
                            if (bb < p.batch && row < p.n) {
                                if (p.y_dtype == BQ_F32)
                                    static_cast<float*>(p.y)[bb * p.n + row] = yacc[j][nt][r];
                                else
                                    static_cast<uint16_t*>(p.y)[bb * p.n + row] = float_to_bf16_bits(yacc[j][nt][r]);
                            }
                        }
            }
        } else {
            const int slot_p = (item_begin(c, T, C) / S == rb) ? 0 : 1;
            float* mine = p.partial + ((c * 2 + slot_p) * p.batch) * kRowsPerCta;
            if (writer) {
#pragma unroll
                for (int j = 0; j < kRowTiles; ++j)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int r = 0; r < 2; ++r) {
                            const int bb = nt * 2 + (t >> 1);
                            if (bb < p.batch)
                                mine[bb * kRowsPerCta + warp * (16 * kRowTiles) + j * 16 + g + 8 * r] = yacc[j][nt][r];
                        }
            }
            __threadfence();
            named_barrier_compute();
            const int64_t c_first = cta_of_item(rb_first, T, C), c_last = cta_of_item(rb_last, T, C);
            if (threadIdx.x == 0) {
                const unsigned int prev = atomicAdd(&p.counters[rb], 1u);
                s_last = (prev == (unsigned int)(c_last - c_first));
            }
            named_barrier_compute();
            if (s_last) {
                __threadfence();
                for (int i = threadIdx.x; i < kRowsPerCta * p.batch; i += kComputeWarps * 32) {
                    const int bb = i / kRowsPerCta, rin = i % kRowsPerCta;
                    const int64_t row = (int64_t)rb * kRowsPerCta + rin;
                    if (row >= p.n) continue;
                    float acc = 0.0f;
                    for (int64_t cc = c_first; cc <= c_last; ++cc) {
                        const int sl = (item_begin(cc, T, C) / S == rb) ? 0 : 1;
                        acc += __ldcg(p.partial + ((cc * 2 + sl) * p.batch + bb) * kRowsPerCta + rin);
                    }
                    if (p.y_dtype == BQ_F32)
                        static_cast<float*>(p.y)[bb * p.n + row] = acc;
                    else
                        static_cast<uint16_t*>(p.y)[bb * p.n + row] = float_to_bf16_bits(acc);
                }
                if (threadIdx.x == 0) p.counters[rb] = 0u;
            }
        }
#pragma unroll
        for (int j = 0; j < kRowTiles; ++j)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) yacc[j][nt][0] = yacc[j][nt][1] = 0.0f;
    }
}

// ----------------------------------------------------------------- host

struct Plan {
    int nt = 0, stages_total = 0, row_blocks = 0, grid = 0;
    size_t xdata_bytes = 0, counters_off = 0, partial_off = 0, total = 0;
};

bool eligible(int fmt, int64_t n, int64_t k, int batch) {
    return (fmt == BQ_Q1G128 || fmt == BQ_T2G128) && batch >= 1 && batch <= 4 && k > 0 && k % 1024 == 0 &&
           n > 0 && n <= (int64_t)INT32_MAX && k / 8 <= (int64_t)INT32_MAX / 4;
}

Plan make_plan(int fmt, int64_t n, int64_t k, int batch) {
    Plan pl;
    pl.nt = (batch + 1) / 2;
    pl.stages_total = (int)(k / 1024);
    pl.row_blocks = (int)((n + kRowsPerCta - 1) / kRowsPerCta);
    const int ctas_per_sm = 2;
    const int64_t items = (int64_t)pl.row_blocks * pl.stages_total;
    const int64_t cap = (int64_t)sm_count() * ctas_per_sm;
    pl.grid = (int)(items < cap ? items : cap);
    pl.xdata_bytes = (size_t)pl.stages_total * pl.nt * kXTileBytes;
    pl.counters_off = (pl.xdata_bytes + 255) / 256 * 256;
    pl.partial_off = (pl.counters_off + (size_t)pl.row_blocks * 4 + 255) / 256 * 256;
    pl.total = pl.partial_off + (size_t)pl.grid * 2 * batch * kRowsPerCta * 4;
    return pl;
}

template <int FMT, int NT>
cudaError_t launch_typed(const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k, const uint16_t* x,
                         int batch, void* y, int y_dtype, uint8_t* ws, const Plan& pl, cudaStream_t s) {
    using L = Layout<FMT, NT>;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    {
        const cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(gemv_tc_kernel<FMT, NT>), L::kSmemBytes);
        if (e != cudaSuccess) return e;
    }
    const int64_t row_bytes = (FMT == BQ_Q1G128) ? k / 8 : k / 4;
    const int64_t G = k / 128;
    CUtensorMap tm_codes, tm_scales;
    {
        cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)n};
        cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
        cuuint32_t box[2] = {128, (cuuint32_t)kRowsPerCta};
        cuuint32_t es[2] = {1, 1};
        if (enc(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[2] = {(cuuint64_t)G, (cuuint64_t)n};
        cuuint64_t strides[1] = {(cuuint64_t)(G * 2)};
        cuuint32_t box[2] = {(cuuint32_t)kGroupsPerStage, (cuuint32_t)kRowsPerCta};
        cuuint32_t es[2] = {1, 1};
        if (enc(&tm_scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint16_t*>(scales), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    Params prm;
    prm.xdata = ws;
    prm.counters = reinterpret_cast<unsigned int*>(ws + pl.counters_off);
    prm.partial = reinterpret_cast<float*>(ws + pl.partial_off);
    prm.y = y;
    prm.y_dtype = y_dtype;
    prm.batch = batch;
    prm.n = n;
    prm.stages_total = pl.stages_total;
    prm.row_blocks = pl.row_blocks;
    prm.status = device_status_ptr();
    if (!prm.status) return cudaErrorUnknown;
    // Both kernels are launched as programmatic dependents of whatever precedes
    // them in the stream; each waits (griddepcontrol.wait) before touching data
    // the predecessor may still produce or read.
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.stages_total);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, prep_kernel<FMT, NT>, x, k, batch, ws, prm.counters, pl.row_blocks);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3(pl.grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = L::kSmemBytes;
    e = cudaLaunchKernelEx(&cfg, gemv_tc_kernel<FMT, NT>, tm_codes, tm_scales, prm);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace tc

int64_t gemv_tc_workspace_bytes(int fmt, int64_t n, int64_t k, int batch) {
    if (!tc::eligible(fmt, n, k, batch)) return 0;
    return (int64_t)tc::make_plan(fmt, n, k, batch).total;
}

bool gemv_tc_eligible(int fmt, int64_t n, int64_t k, int batch) { return tc::eligible(fmt, n, k, batch); }

cudaError_t launch_gemv_tc(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                           const uint16_t* x, int batch, void* y, int y_dtype, void* workspace, cudaStream_t s) {
    const tc::Plan pl = tc::make_plan(fmt, n, k, batch);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    if (fmt == BQ_Q1G128) {
        if (pl.nt == 1) return tc::launch_typed<BQ_Q1G128, 1>(codes, scales, n, k, x, batch, y, y_dtype, ws, pl, s);
        return tc::launch_typed<BQ_Q1G128, 2>(codes, scales, n, k, x, batch, y, y_dtype, ws, pl, s);
    }
    if (pl.nt == 1) return tc::launch_typed<BQ_T2G128, 1>(codes, scales, n, k, x, batch, y, y_dtype, ws, pl, s);
    return tc::launch_typed<BQ_T2G128, 2>(codes, scales, n, k, x, batch, y, y_dtype, ws, pl, s);
}

}  // namespace bq
