// Embedding lookup on a low-bit table: out[i][k] = BF16(s * q) of row ids[i]
// ("1-bit Bonsai 8B" notes, section 3 and Table 1: the embedding layer is
// low-bit too -- the step before the first projection of a decode step).
//
// One warp per output row; for each 128-weight group lane l writes weights
// 4l .. 4l+3 (8 bytes of BF16), so each group's 256 output bytes go out in one
// coalesced warp store.  s * q is +-s or 0, exactly representable in FP32; the
// only rounding is FP16 s -> BF16 (round to nearest, ties to even).
#include "bq_internal.cuh"
#include "bq_ptx.cuh"

namespace bq {
namespace {

constexpr int kWarpsPerBlock = 8;

// Code of weight i of a group (0..127): +1 / -1 (binary), or the trit c - 1.
template <int FMT>
__device__ __forceinline__ void group_codes(const uint8_t* g, int lane, int (&q)[4]) {
    if (FMT == BQ_Q1G128 || FMT == BQ_A1G128) {
        const uint32_t nib = (g[lane >> 1] >> (4 * (lane & 1))) & 0xFu;  // weights 4l .. 4l+3
#pragma unroll
        for (int j = 0; j < 4; ++j) q[j] = ((nib >> j) & 1u) ? 1 : -1;
    } else if (FMT == BQ_T2G128) {
        const uint32_t b = g[lane];  // four 2-bit codes c = q + 1
#pragma unroll
        for (int j = 0; j < 4; ++j) q[j] = (int)((b >> (2 * j)) & 3u) - 1;
    } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = 4 * lane + j;           // trit i: byte i / 5, base-3 digit i % 5
            uint32_t v = g[i / 5];
            for (int d = i % 5; d > 0; --d) v /= 3u;
            q[j] = (int)(v % 3u) - 1;
        }
    }
}

// BF16 round-to-nearest-even of an FP64 value v whose magnitude is within the
// FP32 range: truncate to FP32 (toward zero), then round the 16 discarded bits
// with a sticky bit for what the truncation dropped (one rounding in all).
__device__ __forceinline__ uint16_t f64_to_bf16_rn(double v) {
    float t;
    asm("cvt.rz.f32.f64 %0, %1;" : "=f"(t) : "d"(v));
    const bool sticky = (double)t != v;
    const uint32_t u = __float_as_uint(t), mag = u & 0x7FFFFFFFu, low = mag & 0xFFFFu;
    uint32_t hi = mag >> 16;
    if (low > 0x8000u || (low == 0x8000u && (sticky || (hi & 1u)))) ++hi;
    return (uint16_t)(((u >> 16) & 0x8000u) | hi);
}

template <int FMT>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    embed_rows_kernel(const uint8_t* __restrict__ codes, const uint16_t* __restrict__ scales, int64_t n, int64_t k,
                      const int32_t* __restrict__ ids, int64_t count, uint16_t* __restrict__ out, int* status) {
    ptx::pdl_launch_dependents();
    ptx::pdl_wait();  // the ids and the table may come from the previous kernel
    const int64_t i = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (i >= count) return;
    const int64_t G = k / 128;
    constexpr bool kBits = FMT == BQ_Q1G128 || FMT == BQ_A1G128;
    const int64_t row_bytes = kBits ? k / 8 : FMT == BQ_T2G128 ? k / 4 : G * 26;
    constexpr int kGroupBytes = kBits ? 16 : FMT == BQ_T2G128 ? 32 : 26;
    const int32_t id = __ldg(ids + i);
    uint2* orow = reinterpret_cast<uint2*>(out + i * k);
    if (id < 0 || (int64_t)id >= n) {
        // an id outside the table: a zero row, reported by bq_check
        for (int64_t g = 0; g < G; ++g) orow[g * 32 + lane] = make_uint2(0u, 0u);
        if (lane == 0) record_status(status, BQ_ERR_SHAPE);
        return;
    }
    const uint8_t* row = codes + (int64_t)id * row_bytes;
    if (FMT == BQ_A1G128) {
        // s b + z (exact in FP64), rounded once to BF16
        const uint32_t* prow = reinterpret_cast<const uint32_t*>(scales) + (int64_t)id * G;
        for (int64_t g = 0; g < G; ++g) {
            const uint32_t pz = __ldg(prow + g);
            const double sv = half_bits_to_float((uint16_t)(pz & 0xFFFFu)), zv = half_bits_to_float((uint16_t)(pz >> 16));
            const uint32_t nib = (row[g * 16 + (lane >> 1)] >> (4 * (lane & 1))) & 0xFu;
            uint32_t o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) o[j] = f64_to_bf16_rn(((nib >> j) & 1u) ? sv + zv : zv);
            orow[g * 32 + lane] = make_uint2(o[0] | (o[1] << 16), o[2] | (o[3] << 16));
        }
        return;
    }
    const uint16_t* srow = scales + (int64_t)id * G;
    for (int64_t g = 0; g < G; ++g) {
        const float s = half_bits_to_float(__ldg(srow + g));
        int q[4];
        group_codes<FMT>(row + g * kGroupBytes, lane, q);
        uint32_t w[2];
#pragma unroll
        for (int h = 0; h < 2; ++h)
            w[h] = (uint32_t)float_to_bf16_bits(s * (float)q[2 * h]) |
                   ((uint32_t)float_to_bf16_bits(s * (float)q[2 * h + 1]) << 16);
        orow[g * 32 + lane] = make_uint2(w[0], w[1]);
    }
}

}  // namespace

cudaError_t launch_embed_rows(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                              const int32_t* ids, int64_t count, uint16_t* out, cudaStream_t s) {
    int* status = device_status_ptr();
    if (!status) return cudaErrorUnknown;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((count + kWarpsPerBlock - 1) / kWarpsPerBlock));
    cfg.blockDim = dim3(kWarpsPerBlock * 32);
    cfg.stream = s;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (fmt == BQ_A1G128)
        e = cudaLaunchKernelEx(&cfg, embed_rows_kernel<BQ_A1G128>, codes, scales, n, k, ids, count, out, status);
    else if (fmt == BQ_Q1G128)
        e = cudaLaunchKernelEx(&cfg, embed_rows_kernel<BQ_Q1G128>, codes, scales, n, k, ids, count, out, status);
    else if (fmt == BQ_T2G128)
        e = cudaLaunchKernelEx(&cfg, embed_rows_kernel<BQ_T2G128>, codes, scales, n, k, ids, count, out, status);
    else
        e = cudaLaunchKernelEx(&cfg, embed_rows_kernel<BQ_T5P8G128>, codes, scales, n, k, ids, count, out, status);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace bq
