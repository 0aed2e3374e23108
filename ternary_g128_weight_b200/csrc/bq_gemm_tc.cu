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
// CTA (one per SM, persistent), tile = 128 weight rows x 256 tokens, K in
// stages of 64 (one 128-byte swizzle row of FP16):
//   warps 0-3 : dequantise the tile's 128 weight rows into the stage's A
//               buffer (K-major, 128-byte swizzle, the UMMA canonical layout);
//   warp 4    : TMA loads of the FP16 activation tile (same layout) into B;
//   warp 5    : allocates TMEM (2 x 256 columns) and issues
//               tcgen05.mma.kind::f16 (M = 128, N = 256, K = 16);
//   warps 6-9 : epilogue: TMEM -> registers -> x 2^-e_t -> BF16 -> Y, while
//               the MMAs of the next tile accumulate in the other buffer.
// Tiles are taken token-tile-major so that the activation tile in flight and
// the packed weights stay resident in L2.
#include <cuda.h>

#include "bq_internal.cuh"
#include "bq_ptx.cuh"

namespace bq {
namespace gemm {

constexpr int kTileM = 128;   // weight rows
constexpr int kTileN = 256;   // tokens
constexpr int kStageK = 64;   // FP16 K per stage = 128 bytes per row
constexpr int kStages = 4;
constexpr int kABytes = kTileM * kStageK * 2;  // 16 KB
constexpr int kBBytes = kTileN * kStageK * 2;  // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kDequantWarps = 4, kTmaWarp = 4, kMmaWarp = 5, kEpiWarp0 = 6, kEpiWarps = 4;
constexpr int kThreads = (kEpiWarp0 + kEpiWarps) * 32;
constexpr int kTmemCols = 2 * kTileN;
constexpr int kBarriers = 3 * kStages + 4;
constexpr int kSmemBytes = kStages * kStageBytes + 1024 + kBarriers * 8 + 16;
constexpr uint32_t kWaitPolls = 1u << 24;

struct Params {
    const uint8_t* codes;
    const uint16_t* scales;
    const float* inv_scale;  // [T] 2^-e_t
    uint16_t* y;             // [T][N] BF16
    int64_t n, k, t;
    int fmt;
    int* status;
};

// ----------------------------------------------------------------- X prep
// One CTA per token: X' = FP16(x * 2^e), inv_scale = 2^-e with
// e = 14 - floor(log2 max|x|) (0 for an all-zero row).
__global__ void __launch_bounds__(256) xprep_f16_kernel(const uint16_t* __restrict__ x, int64_t k,
                                                        uint16_t* __restrict__ xh, float* __restrict__ inv_scale) {
    __shared__ float s_max[8];
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
    m = s_max[0];
    for (int i = 1; i < 8; ++i) m = fmaxf(m, s_max[i]);
    int e = (m > 0.f) ? 14 - ilogbf(m) : 0;
    e = max(-126, min(126, e));
    if (threadIdx.x == 0) inv_scale[t] = ldexpf(1.0f, -e);
    uint16_t* out = xh + t * k;
    for (int64_t i = threadIdx.x * 8; i < k; i += blockDim.x * 8) {
        const uint4 v = *reinterpret_cast<const uint4*>(row + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __half lo = __float2half_rn(ldexpf(bf16_lo(w[j]), e));
            const __half hi = __float2half_rn(ldexpf(bf16_hi(w[j]), e));
            o[j] = (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
        }
        *reinterpret_cast<uint4*>(out + i) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// ----------------------------------------------------------------- dequant
// The packed bytes and the scale of 64 weights of one row (k0 .. k0+63).
// Loaded several stages ahead of their use so that the load latency overlaps
// the dequantisation and the MMAs of the stages in between.
struct RowChunk {
    uint4 codes;     // binary: 8 bytes; 2-bit: 16 bytes; 5-per-byte: 14 bytes from an even offset
    uint32_t scale;  // FP16 bits (0 for rows past the end)
};

template <int FMT>
__device__ __forceinline__ RowChunk load_chunk(const Params& p, int64_t row, int64_t k0) {
    RowChunk c;
    c.codes = make_uint4(0u, 0u, 0u, 0u);
    c.scale = 0u;
    if (row >= p.n) return c;
    const int64_t G = p.k / 128;
    c.scale = __ldg(p.scales + row * G + (k0 >> 7));
    if (FMT == BQ_Q1G128) {
        const uint2 b = __ldg(reinterpret_cast<const uint2*>(p.codes + row * (p.k / 8) + (k0 >> 3)));
        c.codes = make_uint4(b.x, b.y, 0u, 0u);
    } else if (FMT == BQ_T2G128) {
        c.codes = __ldg(reinterpret_cast<const uint4*>(p.codes + row * (p.k / 4) + (k0 >> 2)));
    } else {
        // trits 64h .. 64h+63 of the group live in bytes 12h .. 12h+13 (even offset)
        const uint16_t* src =
            reinterpret_cast<const uint16_t*>(p.codes + row * (26 * G) + (k0 >> 7) * 26 + ((k0 & 127) ? 12 : 0));
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

// Base-3 digits of trits BASE .. BASE+63 of a group (5 per byte, least
// significant first) from the bytes load_chunk fetched.
template <int BASE>
__device__ __forceinline__ void t5p8_codes(const RowChunk& c, uint32_t (&code)[64]) {
    const uint32_t wv[4] = {c.codes.x, c.codes.y, c.codes.z, c.codes.w};
    constexpr int kByte0 = BASE ? 12 : 0;  // first loaded byte
#pragma unroll
    for (int i = 0; i < 64; ++i) {
        const int kk = BASE + i, j = kk / 5 - kByte0, d = kk % 5;
        uint32_t v = (wv[j >> 2] >> (8 * (j & 3))) & 0xFFu;
        // floor(v / 3^d) by multiply-shift (exact for v < 256), then mod 3
#pragma unroll
        for (int e = 0; e < d; ++e) v = (v * 171u) >> 9;
        code[i] = v - 3u * ((v * 171u) >> 9);
    }
}

// 64 weights -> 32 FP16 pairs s*q.
template <int FMT>
__device__ __forceinline__ void dequant_chunk(const RowChunk& c, int64_t k0, uint32_t (&h)[32]) {
    const uint32_t s = c.scale;
    const uint32_t ss = s | (s << 16);
    if (FMT == BQ_Q1G128) {
        // bit 1 -> +s, bit 0 -> -s: flip the FP16 sign where the bit is 0
        const uint32_t nb[2] = {~c.codes.x, ~c.codes.y};
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const uint32_t w = nb[i >> 4];
            const int j = 2 * (i & 15);
            h[i] = ss ^ (((w >> j) & 1u) << 15) ^ (((w >> (j + 1)) & 1u) << 31);
        }
    } else {
        // code c in {0, 1, 2} -> -s, 0, +s: magnitude s unless c == 1, sign when c == 0
        uint32_t code[64];
        if (FMT == BQ_T2G128) {
            const uint32_t wv[4] = {c.codes.x, c.codes.y, c.codes.z, c.codes.w};
#pragma unroll
            for (int i = 0; i < 64; ++i) code[i] = (wv[i >> 4] >> (2 * (i & 15))) & 3u;
        } else if ((k0 & 127) == 0) {
            t5p8_codes<0>(c, code);
        } else {
            t5p8_codes<64>(c, code);
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const uint32_t c0 = code[2 * i], c1 = code[2 * i + 1];
            const uint32_t lo = (c0 == 1u) ? 0u : (s | ((c0 == 0u) ? 0x8000u : 0u));
            const uint32_t hi = (c1 == 1u) ? 0u : (s | ((c1 == 0u) ? 0x8000u : 0u));
            h[i] = lo | (hi << 16);
        }
    }
}

// ----------------------------------------------------------------- main
template <int FMT>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_x,
                                                              const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full_a = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
    uint64_t* full_b = full_a + kStages;
    uint64_t* empty = full_b + kStages;
    uint64_t* acc_full = empty + kStages;
    uint64_t* acc_empty = acc_full + 2;
    uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(acc_empty + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t mb_count = (p.n + kTileM - 1) / kTileM, nb_count = (p.t + kTileN - 1) / kTileN;
    const int64_t tiles = mb_count * nb_count;
    const int stages_per_tile = (int)(p.k / kStageK);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            ptx::mbar_init(&full_a[i], kDequantWarps);
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
        const int r = warp * 32 + lane;
        const int64_t my_tiles = (tiles > blockIdx.x) ? (tiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
        const int64_t total = my_tiles * stages_per_tile;
        // the chunk of stage g of this CTA's sequence (tile-major, then K)
        auto chunk_of = [&](int64_t g) {
            const int64_t tile = blockIdx.x + (g / stages_per_tile) * gridDim.x;
            const int64_t st = g % stages_per_tile;
            return load_chunk<FMT>(p, (tile % mb_count) * kTileM + r, st * kStageK);
        };
        constexpr int kAhead = 3;
        RowChunk pipe[kAhead];
#pragma unroll
        for (int i = 0; i < kAhead; ++i) pipe[i] = (i < total) ? chunk_of(i) : RowChunk{};
        for (int64_t it = 0; it < total; ++it) {
            const RowChunk cur = pipe[0];
#pragma unroll
            for (int i = 0; i < kAhead - 1; ++i) pipe[i] = pipe[i + 1];
            if (it + kAhead < total) pipe[kAhead - 1] = chunk_of(it + kAhead);
            const int slot = (int)(it % kStages);
            if (it >= kStages &&
                !ptx::mbar_wait_bounded(&empty[slot], (uint32_t)(((it / kStages) - 1) & 1), kWaitPolls)) {
                record_status(p.status, BQ_ERR_TIMEOUT);
                break;
            }
            uint32_t h[32];
            dequant_chunk<FMT>(cur, (it % stages_per_tile) * kStageK, h);
            uint8_t* a = smem + slot * kStageBytes + r * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4*>(a + ((c ^ (r & 7)) << 4)) =
                    make_uint4(h[4 * c], h[4 * c + 1], h[4 * c + 2], h[4 * c + 3]);
            ptx::fence_proxy_async_smem();  // generic-proxy stores -> visible to the tensor core
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&full_a[slot]);
        }
    } else if (warp == kTmaWarp) {
        // ------------------------------------------------ activation TMA
        if (lane == 0) {
            ptx::prefetch_tensormap(&tm_x);
            int64_t it = 0;
            bool alive = true;
            for (int64_t tile = blockIdx.x; tile < tiles && alive; tile += gridDim.x) {
                const int64_t nb = tile / mb_count;
                for (int st = 0; st < stages_per_tile; ++st, ++it) {
                    const int slot = (int)(it % kStages);
                    if (it >= kStages &&
                        !ptx::mbar_wait_bounded(&empty[slot], (uint32_t)(((it / kStages) - 1) & 1), kWaitPolls)) {
                        record_status(p.status, BQ_ERR_TIMEOUT);
                        alive = false;
                        break;
                    }
                    ptx::mbar_arrive_expect_tx(&full_b[slot], kBBytes);
                    ptx::tma_load_2d(smem + slot * kStageBytes + kABytes, &tm_x, st * kStageK, (int32_t)(nb * kTileN),
                                     &full_b[slot]);
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
            // D f32, A f16, B f16, both K-major, N = 256, M = 128
            const uint32_t idesc = (1u << 4) | ((uint32_t)(kTileN >> 3) << 17) | (8u << 24);
            int64_t it = 0, local = 0;
            bool ok = true;
            for (int64_t tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++local) {
                const int ab = (int)(local & 1);
                if (local >= 2 &&
                    !ptx::mbar_wait_bounded(&acc_empty[ab], (uint32_t)(((local >> 1) - 1) & 1), kWaitPolls)) {
                    record_status(p.status, BQ_ERR_TIMEOUT);
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                for (int st = 0; st < stages_per_tile; ++st, ++it) {
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
                        ptx::mma_f16_ss(tmem + ab * kTileN, ad, bd, idesc, (st > 0 || kk > 0) ? 1u : 0u);
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
        for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++local) {
            const int ab = (int)(local & 1);
            const int64_t mb = tile % mb_count, nb = tile / mb_count;
            if (!ptx::mbar_wait_bounded(&acc_full[ab], (uint32_t)((local >> 1) & 1), kWaitPolls)) {
                record_status(p.status, BQ_ERR_TIMEOUT);
                break;
            }
            ptx::tc_fence_after();
            const int64_t row = mb * kTileM + r;
#pragma unroll 1
            for (int c0 = 0; c0 < kTileN; c0 += 32) {
                uint32_t v[32];
                ptx::tmem_ld_x32(tmem + lane_base + ab * kTileN + c0, v);
                ptx::tc_wait_ld();
                const int64_t t0 = nb * kTileN + c0;
                if (row < p.n) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int64_t tok = t0 + j;
                        if (tok < p.t)
                            p.y[tok * p.n + row] = float_to_bf16_bits(__uint_as_float(v[j]) * __ldg(p.inv_scale + tok));
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

template <int FMT>
cudaError_t launch_typed(const Params& prm, const uint16_t* x, uint16_t* xh, float* inv_scale, cudaStream_t s) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    CUtensorMap tm_x;
    {
        cuuint64_t dims[2] = {(cuuint64_t)prm.k, (cuuint64_t)prm.t};
        cuuint64_t strides[1] = {(cuuint64_t)(prm.k * 2)};
        cuuint32_t box[2] = {(cuuint32_t)kStageK, (cuuint32_t)kTileN};
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
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, xprep_f16_kernel, x, (int64_t)prm.k, xh, inv_scale);
    if (e != cudaSuccess) return e;
    const int64_t tiles = ((prm.n + kTileM - 1) / kTileM) * ((prm.t + kTileN - 1) / kTileN);
    const int64_t grid = tiles < sm_count() ? tiles : sm_count();
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    e = cudaLaunchKernelEx(&cfg, gemm_tc_kernel<FMT>, tm_x, prm);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace gemm

// Workspace of the tensor-core GEMM: FP16 activations [T][K] + inverse
// pre-scales [T] (256-byte aligned pieces).
int64_t gemm_tc_workspace_bytes(int64_t n, int64_t k, int64_t t) {
    (void)n;
    const int64_t xh = (t * k * 2 + 255) / 256 * 256;
    return xh + (t * 4 + 255) / 256 * 256;
}

bool gemm_tc_eligible(int fmt, int64_t n, int64_t k, int64_t t) {
    return (fmt == BQ_Q1G128 || fmt == BQ_T2G128 || fmt == BQ_T5P8G128) && n > 0 && k > 0 && k % 128 == 0 &&
           t > 0 && t <= (int64_t)INT32_MAX && n <= (int64_t)INT32_MAX && (k * 2) % 16 == 0;
}

cudaError_t launch_gemm_tc(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                           const uint16_t* x, int64_t t, uint16_t* y, void* workspace, cudaStream_t s) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint16_t* xh = reinterpret_cast<uint16_t*>(ws);
    float* inv = reinterpret_cast<float*>(ws + (t * k * 2 + 255) / 256 * 256);
    gemm::Params prm;
    prm.codes = codes;
    prm.scales = scales;
    prm.inv_scale = inv;
    prm.y = y;
    prm.n = n;
    prm.k = k;
    prm.t = t;
    prm.fmt = fmt;
    prm.status = device_status_ptr();
    if (!prm.status) return cudaErrorUnknown;
    if (fmt == BQ_Q1G128) return gemm::launch_typed<BQ_Q1G128>(prm, x, xh, inv, s);
    if (fmt == BQ_T2G128) return gemm::launch_typed<BQ_T2G128>(prm, x, xh, inv, s);
    return gemm::launch_typed<BQ_T5P8G128>(prm, x, xh, inv, s);
}

}  // namespace bq
