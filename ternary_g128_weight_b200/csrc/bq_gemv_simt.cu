// Plain CUDA-core GEMV for every format and batch 1..16.  One warp per output
// row; lane l takes the row's groups l, l+32, ...; codes are decoded in
// registers, each group's partial sum is taken in FP32 and multiplied once by
// the group scale, and the lanes' sums are combined with a warp shuffle tree.
// It is the general path (any K % 128 == 0, any alignment of t5p8 rows) and the
// baseline the tensor-core decode path is measured against.
// Pages: "1-bit Bonsai 8B" notes section 4.1 (codes decoded inline in the
// matmul; effective weight = signed code x group FP16 scale).
#include "bq_internal.cuh"

namespace bq {
namespace {

template <int B>
__device__ __forceinline__ void add_word_q1(uint32_t w, const uint16_t* __restrict__ x, int64_t k,
                                            int64_t k0, float (&p)[B]) {
    // 32 consecutive weights k0..k0+31, bit i -> weight k0+i
#pragma unroll
    for (int c = 0; c < 4; ++c) {  // 8 weights per 16-byte load of x
#pragma unroll
        for (int b = 0; b < B; ++b) {
            const uint4 xv = __ldg(reinterpret_cast<const uint4*>(x + b * k + k0 + 8 * c));
            const uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i0 = 8 * c + 2 * e;
                const float x0 = bf16_lo(xs[e]), x1 = bf16_hi(xs[e]);
                p[b] += ((w >> i0) & 1u) ? x0 : -x0;
                p[b] += ((w >> (i0 + 1)) & 1u) ? x1 : -x1;
            }
        }
    }
}

template <int B>
__device__ __forceinline__ void add_word_t2(uint32_t w, const uint16_t* __restrict__ x, int64_t k,
                                            int64_t k0, float (&p)[B]) {
    // 16 consecutive trits k0..k0+15, code c at bits 2i: trit = c - 1
#pragma unroll
    for (int c = 0; c < 2; ++c) {
#pragma unroll
        for (int b = 0; b < B; ++b) {
            const uint4 xv = __ldg(reinterpret_cast<const uint4*>(x + b * k + k0 + 8 * c));
            const uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i0 = 8 * c + 2 * e;
                const float t0 = (float)((int)((w >> (2 * i0)) & 3u) - 1);
                const float t1 = (float)((int)((w >> (2 * i0 + 2)) & 3u) - 1);
                p[b] = fmaf(t0, bf16_lo(xs[e]), p[b]);
                p[b] = fmaf(t1, bf16_hi(xs[e]), p[b]);
            }
        }
    }
}

template <int FMT, int B>
__global__ void __launch_bounds__(256) gemv_simt_kernel(const uint8_t* __restrict__ codes,
                                                        const uint16_t* __restrict__ scales,
                                                        int64_t n, int64_t k,
                                                        const uint16_t* __restrict__ x, void* y,
                                                        int y_dtype) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= n) return;
    const int64_t G = k / kGroup;
    float acc[B];
#pragma unroll
    for (int b = 0; b < B; ++b) acc[b] = 0.0f;

    for (int64_t g = lane; g < G; g += 32) {
        const float s = half_bits_to_float(__ldg(scales + row * G + g));
        float p[B];
#pragma unroll
        for (int b = 0; b < B; ++b) p[b] = 0.0f;
        const int64_t kbase = g * kGroup;
        if (FMT == BQ_Q1G128) {
            const uint4 cw = __ldg(reinterpret_cast<const uint4*>(codes + row * (k / 8) + g * 16));
            add_word_q1<B>(cw.x, x, k, kbase + 0, p);
            add_word_q1<B>(cw.y, x, k, kbase + 32, p);
            add_word_q1<B>(cw.z, x, k, kbase + 64, p);
            add_word_q1<B>(cw.w, x, k, kbase + 96, p);
        } else if (FMT == BQ_T2G128) {
            const uint4* src = reinterpret_cast<const uint4*>(codes + row * (k / 4) + g * 32);
            const uint4 c0 = __ldg(src), c1 = __ldg(src + 1);
            add_word_t2<B>(c0.x, x, k, kbase + 0, p);
            add_word_t2<B>(c0.y, x, k, kbase + 16, p);
            add_word_t2<B>(c0.z, x, k, kbase + 32, p);
            add_word_t2<B>(c0.w, x, k, kbase + 48, p);
            add_word_t2<B>(c1.x, x, k, kbase + 64, p);
            add_word_t2<B>(c1.y, x, k, kbase + 80, p);
            add_word_t2<B>(c1.z, x, k, kbase + 96, p);
            add_word_t2<B>(c1.w, x, k, kbase + 112, p);
        } else {
            const uint8_t* src = codes + row * (G * 26) + g * 26;
#pragma unroll 1
            for (int j = 0; j < 26; ++j) {
                uint32_t v = __ldg(src + j);
                const int nt = (j < 25) ? 5 : 3;
                for (int i = 0; i < nt; ++i) {
                    const float t = (float)((int)(v % 3u) - 1);
                    v /= 3u;
                    const int64_t kk = kbase + 5 * j + i;
#pragma unroll
                    for (int b = 0; b < B; ++b)
                        p[b] = fmaf(t, bf16_bits_to_float(__ldg(x + b * k + kk)), p[b]);
                }
            }
        }
#pragma unroll
        for (int b = 0; b < B; ++b) acc[b] = fmaf(s, p[b], acc[b]);
    }
#pragma unroll
    for (int b = 0; b < B; ++b) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc[b] += __shfl_xor_sync(0xffffffffu, acc[b], off);
    }
    if (lane == 0) {
#pragma unroll
        for (int b = 0; b < B; ++b) {
            if (y_dtype == BQ_F32)
                static_cast<float*>(y)[b * n + row] = acc[b];
            else
                static_cast<uint16_t*>(y)[b * n + row] = float_to_bf16_bits(acc[b]);
        }
    }
}

template <int FMT, int B>
cudaError_t launch_fb(const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                      const uint16_t* x, void* y, int y_dtype, cudaStream_t s) {
    const int64_t blocks = (n + 7) / 8;
    gemv_simt_kernel<FMT, B><<<(unsigned)blocks, 256, 0, s>>>(codes, scales, n, k, x, y, y_dtype);
    return cudaGetLastError();
}

template <int FMT>
cudaError_t launch_f(const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                     const uint16_t* x, int batch, void* y, int y_dtype, cudaStream_t s) {
    switch (batch) {
#define BQ_CASE(BB) case BB: return launch_fb<FMT, BB>(codes, scales, n, k, x, y, y_dtype, s);
        BQ_CASE(1) BQ_CASE(2) BQ_CASE(3) BQ_CASE(4) BQ_CASE(5) BQ_CASE(6) BQ_CASE(7) BQ_CASE(8)
        BQ_CASE(9) BQ_CASE(10) BQ_CASE(11) BQ_CASE(12) BQ_CASE(13) BQ_CASE(14) BQ_CASE(15) BQ_CASE(16)
#undef BQ_CASE
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_gemv_simt(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n,
                             int64_t k, const uint16_t* x, int batch, void* y, int y_dtype,
                             cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    if (fmt == BQ_Q1G128) return launch_f<BQ_Q1G128>(codes, scales, n, k, x, batch, y, y_dtype, s);
    if (fmt == BQ_T2G128) return launch_f<BQ_T2G128>(codes, scales, n, k, x, batch, y, y_dtype, s);
    return launch_f<BQ_T5P8G128>(codes, scales, n, k, x, batch, y, y_dtype, s);
}

}  // namespace bq
