// Packers: float W -> codes + FP16 group scales, one thread per 128-weight
// group.  Pages: "Bonsai-27B-mlx-1bit ... Binary g128" (sign bit, 0 -> -scale,
// 1 -> +scale, FP16 scale per 128 weights); "Ternary Bonsai" (trits times FP16
// group scale); "把 27B 模型压到 4GB" section 2.4 (2-bit slots; five trits per
// byte).  The scale and threshold rules are readings (the pages give weights
// already trained): s = FP16_RNE(mean |w| summed in order in FP64), binary
// q = (w >= 0 ? +1 : -1), ternary q = (|w| <= s/2 ? 0 : sign w).  The FP64
// sum runs in the same order as the definition, so the result is bit-exact.
#include "bq_internal.cuh"

namespace bq {
namespace {

__device__ __forceinline__ uint16_t f64_to_f16_rn(double v) {
    unsigned short h;
    asm("cvt.rn.f16.f64 %0, %1;" : "=h"(h) : "d"(v));
    return h;
}

__device__ __forceinline__ double f16_bits_to_f64(uint16_t h) {
    float f;
    asm("cvt.f32.f16 %0, %1;" : "=f"(f) : "h"(h));
    return (double)f;
}

template <int FMT>
__global__ void __launch_bounds__(128) pack_kernel(const float* __restrict__ w, int64_t n,
                                                   int64_t k, const uint16_t* __restrict__ scales_in,
                                                   uint8_t* __restrict__ codes,
                                                   uint16_t* __restrict__ scales,
                                                   unsigned long long* first_error) {
    const int64_t G = k / kGroup;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= n * G) return;
    const int64_t r = gid / G, g = gid - r * G;
    const float4* src = reinterpret_cast<const float4*>(w + r * k + g * kGroup);

    float v[kGroup];
#pragma unroll
    for (int i = 0; i < kGroup / 4; ++i) {
        float4 f = __ldg(src + i);
        v[4 * i + 0] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
    }
    bool finite = true;
#pragma unroll
    for (int i = 0; i < kGroup; ++i) finite &= isfinite(v[i]);
    if (!finite) { record_pack_error(first_error, gid, BQ_ERR_NONFINITE); return; }

    uint16_t sh;
    if (scales_in) {
        sh = scales_in[r * G + g];
        if ((sh & 0x8000u) || (sh & 0x7C00u) == 0x7C00u) { record_pack_error(first_error, gid, BQ_ERR_SCALE_RANGE); return; }
    } else {
        double sum = 0.0;
#pragma unroll
        for (int i = 0; i < kGroup; ++i) sum = __dadd_rn(sum, fabs((double)v[i]));
        sh = f64_to_f16_rn(sum / 128.0);
        if ((sh & 0x7C00u) == 0x7C00u) { record_pack_error(first_error, gid, BQ_ERR_SCALE_RANGE); return; }
    }
    scales[r * G + g] = sh;
    const double half_s = f16_bits_to_f64(sh) / 2.0;

    if (FMT == BQ_Q1G128) {
        uint32_t word[4] = {0, 0, 0, 0};
#pragma unroll
        for (int i = 0; i < kGroup; ++i)
            if (v[i] >= 0.0f) word[i >> 5] |= 1u << (i & 31);
        uint4* dst = reinterpret_cast<uint4*>(codes + r * (k / 8) + g * 16);
        *dst = make_uint4(word[0], word[1], word[2], word[3]);
    } else if (FMT == BQ_T2G128) {
        uint32_t word[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
        for (int i = 0; i < kGroup; ++i) {
            const double a = fabs((double)v[i]);
            const uint32_t c = (a <= half_s) ? 1u : (v[i] > 0.0f ? 2u : 0u);
            word[i >> 4] |= c << (2 * (i & 15));
        }
        uint4* dst = reinterpret_cast<uint4*>(codes + r * (k / 4) + g * 32);
        dst[0] = make_uint4(word[0], word[1], word[2], word[3]);
        dst[1] = make_uint4(word[4], word[5], word[6], word[7]);
    } else {
        uint8_t* dst = codes + r * (G * 26) + g * 26;
#pragma unroll
        for (int j = 0; j < 26; ++j) {
            uint32_t byte = 0, p3 = 1;
#pragma unroll
            for (int i = 0; i < 5; ++i) {
                const int idx = 5 * j + i;
                if (idx < kGroup) {
                    const double a = fabs((double)v[idx]);
                    const uint32_t c = (a <= half_s) ? 1u : (v[idx] > 0.0f ? 2u : 0u);
                    byte += c * p3;
                }
                p3 *= 3;
            }
            dst[j] = (uint8_t)byte;
        }
    }
}

// Affine 1-bit variant (the layout MLX packs: a scale and a bias per group,
// "Bonsai-27B-mlx-1bit ... Binary g128", section "MLX打包优化").  Reading of
// the rule: z = FP16_RNE(min w), s = FP16_RNE(max w - min w) (exact in FP64),
// bit = 1 iff w - z > s/2 in FP64 (ties give 0); params [N][G][2] = (s, z).
__global__ void __launch_bounds__(128) pack_affine_kernel(const float* __restrict__ w, int64_t n, int64_t k,
                                                          const uint16_t* __restrict__ params_in,
                                                          uint8_t* __restrict__ codes, uint16_t* __restrict__ params,
                                                          unsigned long long* first_error) {
    const int64_t G = k / kGroup;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= n * G) return;
    const int64_t r = gid / G, g = gid - r * G;
    const float4* src = reinterpret_cast<const float4*>(w + r * k + g * kGroup);
    float v[kGroup];
#pragma unroll
    for (int i = 0; i < kGroup / 4; ++i) {
        float4 f = __ldg(src + i);
        v[4 * i + 0] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
    }
    bool finite = true;
#pragma unroll
    for (int i = 0; i < kGroup; ++i) finite &= isfinite(v[i]);
    if (!finite) { record_pack_error(first_error, gid, BQ_ERR_NONFINITE); return; }
    uint16_t sh, zh;
    if (params_in) {
        sh = params_in[2 * gid];
        zh = params_in[2 * gid + 1];
        if ((sh & 0x8000u) || (sh & 0x7C00u) == 0x7C00u || (zh & 0x7C00u) == 0x7C00u) {
            record_pack_error(first_error, gid, BQ_ERR_SCALE_RANGE);
            return;
        }
    } else {
        float lo = v[0], hi = v[0];
#pragma unroll
        for (int i = 1; i < kGroup; ++i) {
            lo = fminf(lo, v[i]);
            hi = fmaxf(hi, v[i]);
        }
        zh = f64_to_f16_rn((double)lo);
        sh = f64_to_f16_rn((double)hi - (double)lo);
        if ((sh & 0x7C00u) == 0x7C00u || (zh & 0x7C00u) == 0x7C00u) {
            record_pack_error(first_error, gid, BQ_ERR_SCALE_RANGE);
            return;
        }
    }
    params[2 * gid] = sh;
    params[2 * gid + 1] = zh;
    const double zv = f16_bits_to_f64(zh), half_s = f16_bits_to_f64(sh) / 2.0;
    uint32_t word[4] = {0, 0, 0, 0};
#pragma unroll
    for (int i = 0; i < kGroup; ++i)
        if ((double)v[i] - zv > half_s) word[i >> 5] |= 1u << (i & 31);
    uint4* dst = reinterpret_cast<uint4*>(codes + r * (k / 8) + g * 16);
    *dst = make_uint4(word[0], word[1], word[2], word[3]);
}

}  // namespace

cudaError_t launch_pack(int fmt, const float* w, int64_t n, int64_t k, const uint16_t* scales_in,
                        uint8_t* codes, uint16_t* scales, unsigned long long* first_error,
                        cudaStream_t s) {
    const int64_t groups = n * (k / kGroup);
    if (groups == 0) return cudaSuccess;
    const int threads = 128;
    const int64_t blocks = (groups + threads - 1) / threads;
    if (fmt == BQ_A1G128)
        pack_affine_kernel<<<(unsigned)blocks, threads, 0, s>>>(w, n, k, scales_in, codes, scales, first_error);
    else if (fmt == BQ_Q1G128)
        pack_kernel<BQ_Q1G128><<<(unsigned)blocks, threads, 0, s>>>(w, n, k, scales_in, codes, scales, first_error);
    else if (fmt == BQ_T2G128)
        pack_kernel<BQ_T2G128><<<(unsigned)blocks, threads, 0, s>>>(w, n, k, scales_in, codes, scales, first_error);
    else
        pack_kernel<BQ_T5P8G128><<<(unsigned)blocks, threads, 0, s>>>(w, n, k, scales_in, codes, scales, first_error);
    return cudaGetLastError();
}

}  // namespace bq
