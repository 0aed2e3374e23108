// Weight-streaming GEMV on the 5th-generation tensor cores (tcgen05): binary
// g128 and 2-bit-slot ternary g128, batch 1..4, K % 1024 == 0.
//
// Why the tensor core at all: at batch 1 the binary format must be consumed at
// ~126 weights per clock per SM to stream HBM at 80% of its bandwidth, while
// the integer/logic pipe retires 64 operations per clock per SM, so a decode
// that spends one instruction per weight cannot keep up (the "1-bit Bonsai 8B"
// notes, section 4.4, observe the same shift of inline dequantisation towards
// compute).  Here the CUDA cores only expand bits with LOP3 (a quarter of an
// instruction per weight) and the multiply-accumulate runs asynchronously on
// the tensor core with the accumulators in tensor memory:
//
//   binary : byte j of (w & (0x01010101 << p)) is 2^p * bit(8j+p) of the
//            32-bit code word w; eight masks turn one word into eight operand
//            columns.  The activation operand of that k-slot is Q_k / 2^p.
//   2-bit  : byte j of ((w >> 2i) & 0x03030303) is the code c = q+1 of trit
//            4j+i of the word; the activation operand is Q_k.
//
// Q is the activation in fixed point: per (batch row b, group g) a power of
// two 2^E maps the group's largest |x| into [2^29, 2^30); Q = round(x 2^E)
// (binary: rounded to a multiple of 2^7 so that Q / 2^p is an integer).  Q is
// split into four signed base-256 digits, one MMA column each (N = 4 * batch
// slots), and the four int32 column sums are recombined in FP32.  Per group g
// and row: binary y += s (2^(1-E) sum_k bit_k Q_k - 2^-E sum_k Q_k); 2-bit
// y += s (2^-E sum_k c_k Q_k - 2^-E sum_k Q_k); i.e. s * sum_k q_k x_k with
// q = 2 bit - 1 ("Bonsai-27B ... Binary g128": 0 -> -scale, 1 -> +scale) or
// q = c - 1.  The only rounding before FP32 is that of x to Q: at most 2^-23
// of the group's largest |x| per element.
//
// CTA roles (one CTA per SM, 128 rows, all 512 TMEM columns):
//   warps 0-15: decode warps, four per TMEM lane quadrant; warp d handles the
//               rows of quadrant d & 3 (one row per thread = TMEM lane) and
//               groups d >> 2 and (d >> 2) + 4 of every stage: it expands the
//               row's codes into the group's 32 TMEM columns (tcgen05.st) and,
//               one stage later, reads the group's int32 sums back
//               (tcgen05.ld) and folds them into y with the scale;
//   warp 16   : TMA producer (codes with 128-byte swizzle, FP16 scales, and a
//               bulk copy of the prepared activation operand per stage);
//   warp 17   : allocates TMEM and issues the MMAs (M = 128, N = 8 or 16,
//               K = 32 per instruction, A from TMEM, B from shared memory).
// Each group has its own A (32 columns) and D (16 columns) slot, so the
// decode of a stage never waits for the MMAs of the same stage.
// The grid is persistent and splits the (row block, stage) items evenly
// ("stream-K"); a row block shared by two CTAs is finished by the last one,
// which adds the partial sums in CTA order (deterministic).  Launches use
// programmatic dependent launch so that a call's weight stream starts while
// the previous kernel in the stream drains.
#include <cuda.h>

#include "bq_internal.cuh"
#include "bq_ptx.cuh"

namespace bq {
namespace tc {

constexpr int kGroupsPerStage = 8;
constexpr int kRowsPerCta = 128;
constexpr int kSubs = 4;                         // decode warps per TMEM lane quadrant
constexpr int kDecodeWarps = 4 * kSubs;          // warp d: quadrant d & 3, sub d >> 2
constexpr int kProducerWarp = kDecodeWarps;
constexpr int kMmaWarp = kDecodeWarps + 1;
constexpr int kThreads = (kDecodeWarps + 2) * 32;
constexpr int kTmemCols = 512;                   // A: 8 groups x 32 columns, D: 8 groups x 16 columns
constexpr int kDCol0 = kGroupsPerStage * 32;
constexpr uint32_t kWaitPolls = 1u << 24;

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

// Prepared activation operand of one stage: B in the canonical K-major
// no-swizzle layout (per MMA: two 16-byte K chunks x NT groups of 8 rows), then
// the per-(group, batch slot) table {2^a, 2^b, 2^-E sum Q, 0} with 2^(a+b) =
// 2^(shift - E).
template <int NT>
struct XTile {
    static constexpr int kBBytes = kGroupsPerStage * 4 * 256 * NT;
    static constexpr int kTabBytes = kGroupsPerStage * 2 * NT * 16;
    static constexpr int kBytes = kBBytes + kTabBytes;
};

template <int FMT, int NT>
struct Layout {
    static constexpr int kCodesBytes = kRowsPerCta * Fmt<FMT>::kRowBytesPerStage;
    static constexpr int kScalesBytes = kRowsPerCta * kGroupsPerStage * 2;
    static constexpr int kXBytes = XTile<NT>::kBytes;
    static constexpr int kStageBytes = (kCodesBytes + kScalesBytes + kXBytes + 1023) / 1024 * 1024;
    // one CTA per SM
    static constexpr int kStages = (FMT == BQ_Q1G128) ? (NT == 1 ? 6 : 5) : (NT == 1 ? 4 : 3);
    static constexpr int kBarriers = 2 * kStages + 2 * kGroupsPerStage + 1;
    static constexpr int kCombineBytes = (kSubs - 1) * kRowsPerCta * 2 * NT * 4;
    static constexpr int kSmemBytes = kStages * kStageBytes + 1024 + kBarriers * 8 + 16 + kCombineBytes;
};

struct Params {
    const uint8_t* xdata;    // prepared activation operands, [stage][XTile]
    float* partial;          // [grid][2][batch][kRowsPerCta]
    unsigned int* counters;  // [row_blocks], zeroed by the prep kernel
    void* y;
    int y_dtype;
    int batch;
    int64_t n;
    int stages_total;
    int row_blocks;
    int* status;
};

// all decode warps / the sub-0 decode warps (the ones that write outputs)
__device__ __forceinline__ void decode_barrier() {
    asm volatile("bar.sync 1, %0;" ::"n"(kDecodeWarps * 32) : "memory");
}
__device__ __forceinline__ void writer_barrier() { asm volatile("bar.sync 2, 128;" ::: "memory"); }

__host__ __device__ __forceinline__ int64_t item_begin(int64_t c, int64_t T, int64_t C) { return c * T / C; }
__device__ __forceinline__ int64_t cta_of_item(int64_t i, int64_t T, int64_t C) { return ((i + 1) * C - 1) / T; }

// Position of weight kk (0..127) of a group in the MMA K order: MMA index and
// byte (k-slot) inside that MMA's 32-byte K slice.
template <int FMT>
__host__ __device__ __forceinline__ void kslot_of(int kk, int& mma, int& kb) {
    if (FMT == BQ_Q1G128) {  // word q = kk/32, bit 8j+p -> column 8q+p, byte j
        mma = kk >> 5;
        const int pp = kk & 7, j = (kk >> 3) & 3;
        kb = 4 * pp + j;
    } else {  // word w = kk/16 (MMA w/2), trit 4j+i -> column 4(w&1)+i, byte j
        const int w = kk >> 4, i = kk & 3, j = (kk >> 2) & 3;
        mma = w >> 1;
        kb = 4 * (4 * (w & 1) + i) + j;
    }
}

// ----------------------------------------------------------------- prep
// One CTA per group (128 threads, one weight position each).  Writes the
// group's B digits and table entries into its stage's XTile.
template <int FMT, int NT>
__global__ void __launch_bounds__(128) prep_kernel(const uint16_t* __restrict__ x, int64_t k, int batch,
                                                   uint8_t* __restrict__ xdata, unsigned int* counters,
                                                   int row_blocks) {
    __shared__ float s_max[4];
    __shared__ long long s_sum[4];
    ptx::pdl_launch_dependents();
    ptx::pdl_wait();
    const int grp = blockIdx.x;
    const int kk = threadIdx.x, warp = kk >> 5, lane = kk & 31;
    if (grp == 0)
        for (int i = threadIdx.x; i < row_blocks; i += blockDim.x) counters[i] = 0u;
    const int st = grp / kGroupsPerStage, G = grp % kGroupsPerStage;
    uint8_t* tile = xdata + (size_t)st * XTile<NT>::kBytes;
    int mma, kb;
    kslot_of<FMT>(kk, mma, kb);
    const int chunk = kb >> 4, byte = kb & 15;
    uint8_t* bbase = tile + (size_t)(G * 4 + mma) * 256 * NT + chunk * NT * 128 + byte;
    for (int bb = 0; bb < 2 * NT; ++bb) {
        const float xv = (bb < batch) ? bf16_bits_to_float(x[bb * k + (int64_t)grp * 128 + kk]) : 0.0f;
        float m = fabsf(xv);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        if (lane == 0) s_max[warp] = m;
        __syncthreads();
        m = fmaxf(fmaxf(s_max[0], s_max[1]), fmaxf(s_max[2], s_max[3]));
        const int E = (m > 0.f) ? 29 - ilogbf(m) : 0;
        int q, b;
        if (FMT == BQ_Q1G128) {
            q = __float2int_rn(ldexpf(xv, E - 7)) * 128;
            b = q >> (kk & 7);  // exact: q is a multiple of 2^7
        } else {
            q = __float2int_rn(ldexpf(xv, E));
            b = q;
        }
        // balanced base-256 digits: rows n = 4 (bb % 2) + digit of 8-row group bb / 2
        uint8_t* dst = bbase + (bb >> 1) * 128 + (4 * (bb & 1)) * 16;
#pragma unroll
        for (int d = 0; d < 3; ++d) {
            const int dg = (int8_t)(b & 0xFF);
            dst[d * 16] = (uint8_t)dg;
            b = (b - dg) >> 8;
        }
        dst[3 * 16] = (uint8_t)b;
        long long sq = q;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
        if (lane == 0) s_sum[warp] = sq;
        __syncthreads();
        if (kk == 0) {
            const long long tot = s_sum[0] + s_sum[1] + s_sum[2] + s_sum[3];
            const int e = Fmt<FMT>::kCoefShift - E;
            const int a = max(-60, min(60, e));
            float4 tab;
            tab.x = ldexpf(1.0f, a);
            tab.y = ldexpf(1.0f, e - a);
            tab.z = (float)ldexp((double)tot, -E);
            tab.w = 0.0f;
            *reinterpret_cast<float4*>(tile + XTile<NT>::kBBytes + (G * 2 * NT + bb) * 16) = tab;
        }
        __syncthreads();
    }
}

// ----------------------------------------------------------------- main
template <int FMT, int NT>
__global__ void __launch_bounds__(kThreads, 1) gemv_tc_kernel(const __grid_constant__ CUtensorMap tm_codes,
                                                              const __grid_constant__ CUtensorMap tm_scales,
                                                              const Params p) {
    using L = Layout<FMT, NT>;
    constexpr int NB = 2 * NT;  // batch slots
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kStages * L::kStageBytes);
    uint64_t* empty = full + L::kStages;
    uint64_t* a_full = empty + L::kStages;
    uint64_t* mma_done = a_full + kGroupsPerStage;
    uint64_t* final_bar = mma_done + kGroupsPerStage;
    uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(final_bar + 1);
    float* combine = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(tmem_base_smem) + 16);
    __shared__ int s_last;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t S = p.stages_total, T = (int64_t)p.row_blocks * S, C = gridDim.x, c = blockIdx.x;
    const int64_t it0 = item_begin(c, T, C), it1 = item_begin(c + 1, T, C);
    const int nit = (int)(it1 - it0);

    if (threadIdx.x == 0) {
        for (int i = 0; i < L::kStages; ++i) {
            ptx::mbar_init(&full[i], 1);
            ptx::mbar_init(&empty[i], kDecodeWarps + 1);
        }
        for (int i = 0; i < kGroupsPerStage; ++i) {
            ptx::mbar_init(&a_full[i], 4);  // the four quadrant warps of the group's sub
            ptx::mbar_init(&mma_done[i], 1);
        }
        ptx::mbar_init(final_bar, 1);
        ptx::fence_barrier_init();
    }
    if (warp == kMmaWarp) ptx::tmem_alloc(tmem_base_smem, kTmemCols);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_base_smem;
    ptx::pdl_launch_dependents();

    if (warp == kProducerWarp) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            ptx::prefetch_tensormap(&tm_codes);
            ptx::prefetch_tensormap(&tm_scales);
            auto issue_weights = [&](int it) {
                const int slot = it % L::kStages;
                uint8_t* sb = smem + slot * L::kStageBytes;
                const int64_t item = it0 + it;
                const int rb = (int)(item / S), st = (int)(item % S);
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
                const int st = (int)((it0 + it) % S);
                ptx::bulk_load(sb + L::kCodesBytes + L::kScalesBytes, p.xdata + (size_t)st * L::kXBytes,
                               L::kXBytes, &full[slot]);
            };
            // weights do not depend on the previous kernel: stream them first
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
            for (int it = (issued > L::kStages ? issued - L::kStages : 0); it < issued; ++it)
                if (!ptx::mbar_wait_bounded(&full[it % L::kStages], (it / L::kStages) & 1, kWaitPolls))
                    record_status(p.status, BQ_ERR_TIMEOUT);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            // D s32, A u8, B s8, both K-major, N = 8 NT, M = 128
            const uint32_t idesc = (2u << 4) | (0u << 7) | (1u << 10) | ((uint32_t)NT << 17) | (8u << 24);
            bool ok = true;
            for (int it = 0; it < nit && ok; ++it) {
                const int slot = it % L::kStages;
                if (!ptx::mbar_wait_bounded(&full[slot], (it / L::kStages) & 1, kWaitPolls)) {
                    record_status(p.status, BQ_ERR_TIMEOUT);
                    ok = false;
                    break;
                }
                const uint32_t b_s = ptx::smem_u32(smem + slot * L::kStageBytes + L::kCodesBytes + L::kScalesBytes);
#pragma unroll
                for (int G = 0; G < kGroupsPerStage; ++G) {
                    if (!ptx::mbar_wait_bounded(&a_full[G], it & 1, kWaitPolls)) {
                        record_status(p.status, BQ_ERR_TIMEOUT);
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint64_t bd = ptx::smem_desc_kmajor_noswizzle(b_s + (G * 4 + q) * 256 * NT, 128 * NT, 128);
                        ptx::mma_i8_ts(tmem + kDCol0 + G * 16, tmem + G * 32 + q * 8, bd, idesc, q > 0 ? 1u : 0u);
                    }
                    ptx::tc_commit(&mma_done[G]);
                }
                if (ok) ptx::tc_commit(&empty[slot]);
            }
            // all MMAs of this CTA finished before TMEM is released
            ptx::tc_commit(final_bar);
            if (!ptx::mbar_wait_bounded(final_bar, 0, kWaitPolls)) record_status(p.status, BQ_ERR_TIMEOUT);
        }
    } else {
        // ------------------------------------------------ decode + epilogue warps
        const int quad = warp & 3, sub = warp >> 2;
        const int row = quad * 32 + lane;  // row in the CTA tile == TMEM lane
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
        float y[NB];
        float c1[2][NB], f2[2][NB], cx[2][NB];  // coefficients of groups sub and sub + 4
#pragma unroll
        for (int b = 0; b < NB; ++b) y[b] = 0.0f;
        bool alive = true;
        bool prev_stage_open = false;  // this warp's groups of the previous stage await their fold

        auto epi_load = [&](int G, uint32_t (&d)[8 * NT]) {
#pragma unroll
            for (int h = 0; h < NT; ++h) {
                uint32_t t8[8];
                ptx::tmem_ld_x8(tmem + lane_base + kDCol0 + G * 16 + 8 * h, t8);
#pragma unroll
                for (int e = 0; e < 8; ++e) d[8 * h + e] = t8[e];
            }
        };
        auto epi_fold = [&](int j, const uint32_t (&d)[8 * NT]) {
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                // columns 4b..4b+3 hold the four digit sums of batch slot b
                const int lo = (int)d[4 * b] + 256 * (int)d[4 * b + 1];
                const int hi = (int)d[4 * b + 2] + 256 * (int)d[4 * b + 3];
                const float v = fmaf((float)hi, 65536.0f, (float)lo);
                y[b] = fmaf(v * c1[j][b], f2[j][b], y[b]) - cx[j][b];
            }
        };

        for (int it = 0; it < nit; ++it) {
            const int slot = it % L::kStages;
            const int64_t item = it0 + it;
            const int rb = (int)(item / S), st = (int)(item % S);
            if (alive && !ptx::mbar_wait_bounded(&full[slot], (it / L::kStages) & 1, kWaitPolls)) {
                record_status(p.status, BQ_ERR_TIMEOUT);
                alive = false;
            }
            if (alive) {
                const uint8_t* stage = smem + slot * L::kStageBytes;
                const uint16_t* scales_s = reinterpret_cast<const uint16_t*>(stage + L::kCodesBytes);
                const uint8_t* tab_s = stage + L::kCodesBytes + L::kScalesBytes + XTile<NT>::kBBytes;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int G = sub + 4 * j;
                    // previous stage's group G: wait for its MMAs, start reading its sums
                    uint32_t d[8 * NT];
                    const bool fold = it > 0 && prev_stage_open;
                    if (it > 0) {
                        if (!ptx::mbar_wait_bounded(&mma_done[G], (it & 1) ^ 1, kWaitPolls)) {
                            record_status(p.status, BQ_ERR_TIMEOUT);
                            alive = false;
                        }
                        if (fold && alive) {
                            ptx::tc_fence_after();
                            epi_load(G, d);
                        }
                    }
                    // decode group G into its 32 TMEM columns
                    uint32_t a[32];
                    if (FMT == BQ_Q1G128) {
                        const uint4 w = *reinterpret_cast<const uint4*>(stage + row * 128 + ((G ^ (row & 7)) << 4));
                        const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int q = 0; q < 4; ++q)
#pragma unroll
                            for (int pp = 0; pp < 8; ++pp) a[8 * q + pp] = wv[q] & (0x01010101u << pp);
                    } else {
                        const uint8_t* box = stage + (G >> 2) * (kRowsPerCta * 128) + row * 128;
                        const int c0 = 2 * (G & 3);
                        const uint4 wa = *reinterpret_cast<const uint4*>(box + ((c0 ^ (row & 7)) << 4));
                        const uint4 wb = *reinterpret_cast<const uint4*>(box + (((c0 + 1) ^ (row & 7)) << 4));
                        const uint32_t wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
                        for (int w8 = 0; w8 < 8; ++w8)
#pragma unroll
                            for (int i = 0; i < 4; ++i) a[4 * w8 + i] = (wv[w8] >> (2 * i)) & 0x03030303u;
                    }
                    ptx::tmem_st_x32(tmem + lane_base + G * 32, a);
                    if (fold && alive) {
                        ptx::tc_wait_ld();
                        epi_fold(j, d);
                    }
                    // coefficients of group G
                    const float s = half_bits_to_float(scales_s[row * kGroupsPerStage + G]);
#pragma unroll
                    for (int b = 0; b < NB; ++b) {
                        const float4 tab = *reinterpret_cast<const float4*>(tab_s + (G * NB + b) * 16);
                        c1[j][b] = s * tab.x;
                        f2[j][b] = tab.y;
                        cx[j][b] = s * tab.z;
                    }
                    ptx::tc_wait_st();
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&a_full[G]);
                }
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&empty[slot]);
            }
            prev_stage_open = true;
            // ---------------------------------------- row block finished here?
            if (st != S - 1 && it != nit - 1) continue;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int G = sub + 4 * j;
                if (alive && !ptx::mbar_wait_bounded(&mma_done[G], it & 1, kWaitPolls)) {
                    record_status(p.status, BQ_ERR_TIMEOUT);
                    alive = false;
                }
                if (alive) {
                    uint32_t d[8 * NT];
                    ptx::tc_fence_after();
                    epi_load(G, d);
                    ptx::tc_wait_ld();
                    epi_fold(j, d);
                }
            }
            prev_stage_open = false;
            // combine the four subs' partial sums of each row (fixed order)
            if (sub > 0) {
#pragma unroll
                for (int b = 0; b < NB; ++b) combine[((sub - 1) * NB + b) * kRowsPerCta + row] = y[b];
            }
            decode_barrier();
            if (sub == 0) {
#pragma unroll
                for (int k2 = 0; k2 < kSubs - 1; ++k2)
#pragma unroll
                    for (int b = 0; b < NB; ++b) y[b] += combine[(k2 * NB + b) * kRowsPerCta + row];
                const int64_t rb_first = (int64_t)rb * S, rb_last = rb_first + S - 1;
                const bool whole = rb_first >= it0 && rb_last < it1;
                const int64_t grow = (int64_t)rb * kRowsPerCta + row;
                if (whole) {
                    if (grow < p.n) {
#pragma unroll
                        for (int b = 0; b < NB; ++b)
                            if (b < p.batch) {
                                if (p.y_dtype == BQ_F32)
                                    static_cast<float*>(p.y)[b * p.n + grow] = y[b];
                                else
                                    static_cast<uint16_t*>(p.y)[b * p.n + grow] = float_to_bf16_bits(y[b]);
                            }
                    }
                } else {
                    const int slot_p = (it0 / S == rb) ? 0 : 1;
                    float* mine = p.partial + ((c * 2 + slot_p) * p.batch) * kRowsPerCta;
#pragma unroll
                    for (int b = 0; b < NB; ++b)
                        if (b < p.batch) mine[b * kRowsPerCta + row] = y[b];
                    writer_barrier();
                    const int64_t c_first = cta_of_item(rb_first, T, C), c_last = cta_of_item(rb_last, T, C);
                    if (threadIdx.x == 0) {
                        __threadfence();
                        const unsigned int prev = atomicAdd(&p.counters[rb], 1u);
                        s_last = (prev == (unsigned int)(c_last - c_first));
                        if (s_last) __threadfence();
                    }
                    writer_barrier();
                    if (s_last && grow < p.n) {
                        for (int b = 0; b < p.batch; ++b) {
                            float acc = 0.0f;
                            for (int64_t cc = c_first; cc <= c_last; ++cc) {
                                const int sl = (item_begin(cc, T, C) / S == rb) ? 0 : 1;
                                acc += __ldcg(p.partial + ((cc * 2 + sl) * p.batch + b) * kRowsPerCta + row);
                            }
                            if (p.y_dtype == BQ_F32)
                                static_cast<float*>(p.y)[b * p.n + grow] = acc;
                            else
                                static_cast<uint16_t*>(p.y)[b * p.n + grow] = float_to_bf16_bits(acc);
                        }
                    }
                    if (s_last && threadIdx.x == 0) p.counters[rb] = 0u;
                }
            }
            decode_barrier();  // combine buffer reusable
#pragma unroll
            for (int b = 0; b < NB; ++b) y[b] = 0.0f;
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
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

struct Plan {
    int nt = 0, stages_total = 0, row_blocks = 0, grid = 0;
    size_t xdata_bytes = 0, counters_off = 0, partial_off = 0, total = 0;
};

bool eligible(int fmt, int64_t n, int64_t k, int batch) {
    return (fmt == BQ_Q1G128 || fmt == BQ_T2G128) && batch >= 1 && batch <= 4 && k > 0 && k % 1024 == 0 &&
           n > 0 && n <= (int64_t)INT32_MAX && k / 8 <= (int64_t)INT32_MAX / 4;
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

Plan make_plan(int fmt, int64_t n, int64_t k, int batch) {
    Plan pl;
    pl.nt = (batch + 1) / 2;
    pl.stages_total = (int)(k / 1024);
    pl.row_blocks = (int)((n + kRowsPerCta - 1) / kRowsPerCta);
    const int64_t items = (int64_t)pl.row_blocks * pl.stages_total;
    const int64_t cap = (int64_t)sm_count();
    pl.grid = (int)(items < cap ? items : cap);
    pl.xdata_bytes = (size_t)pl.stages_total * (pl.nt == 1 ? XTile<1>::kBytes : XTile<2>::kBytes);
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
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(gemv_tc_kernel<FMT, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             L::kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set = true;
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
    // Both kernels are programmatic dependents of whatever precedes them in the
    // stream and wait (griddepcontrol.wait) before touching data that it may
    // still produce or read.
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)G);
    cfg.blockDim = dim3(128);
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
