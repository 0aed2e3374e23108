// 4-bit KV cache for decode attention: the quantiser (bq_kv4_quantize), the
// per-step append (bq_kv4_append) and split-context grouped-query decode
// attention over the quantised cache (bq_kv4_attention_decode).
//
// Pages: "Bonsai-27B-mlx-1bit ... Binary g128", sections "峰值内存管理" and
// "KV压缩潜力" (a 4-bit KV cache is what keeps long contexts small);
// "Ternary Bonsai", hybrid-attention section (4-bit KV-cache quantisation);
// "1-bit Bonsai 8B" notes, Table 1 (grouped-query attention, 32 query / 8 KV
// heads of dimension 128).
//
// Format (the pages fix only the bit width): every cached K or V vector is cut
// into groups of 128 values; a group is 64 bytes of 4-bit codes (value 2i in
// the low nibble of byte i) plus one 32-bit word (FP16 scale s in the low half,
// FP16 bias z in the high half), quantised min-max affine:
//   s = FP16(RNE((max - min) / 15)),  z = FP16(RNE(min)),
//   c = clamp(rint((x - z) / s), 0, 15)  (0 when s == 0),   value = s c + z.
//
// Attention design (HBM bound: 68 bytes per 128-value vector and per token):
//  * a CTA owns one (sequence, KV head) and a range of the context; its 8 warps
//    take interleaved stages of 8192 / D tokens, each warp with its own ring of
//    three stages fed by 1-D bulk copies (K codes, V codes, K params, V params);
//  * scores: mma.m16n8k32 (u8 x s8 -> s32) with A = the K codes of 16 tokens
//    (even / odd nibbles of a word masked into bytes: 3 instructions per 8
//    values) and B = the group's query heads (up to 8) as 22-bit fixed point in
//    three int8 digit planes, so Σ q c is exact in int32; per token and group the
//    score is s Σ q c + z Σ q;
//  * online softmax in the log2 domain, per head, once per stage;
//  * P V: mma.m16n8k16 with A = V^T codes (the nibbles of two tokens paired by
//    one PRMT) and B = P s_V 2^σ as FP16 (s_V folded into the weights, σ a
//    per-warp power of two that keeps P s_V 2^σ < 2^15), transposed from the
//    score fragment by movmatrix; the bias part Σ p (z + 8 s) is summed apart;
//  * warps merge in shared memory, CTAs of the same (sequence, KV head) through
//    a workspace of partials merged by the last CTA to finish, in split order
//    (deterministic).
#include "bq_internal.cuh"
#include "bq_ptx.cuh"

#include <math.h>

namespace bq {
namespace kv4 {
namespace {

constexpr int kWarps = 8;  // warps per CTA
constexpr int kRing = 3;   // stages in flight per warp
constexpr int kMaxHeads = 8;
constexpr int kNoSigma = 40;  // sigma before any V scale was seen (above every real value)
constexpr uint32_t kWaitPolls = 1u << 23;
constexpr int kAlignSlack = 128;

template <int D>
struct Geo {
    static constexpr int NG = D / 128;          // 128-value groups per vector
    static constexpr int TS = 8192 / D;         // tokens per stage
    static constexpr int MT = TS / 16;          // 16-token tiles per stage
    static constexpr int ROWB = D / 2;          // code bytes per token
    static constexpr int CODEB = TS * ROWB;     // code bytes per stage (4096)
    static constexpr int PARB = TS * NG * 4;    // parameter bytes per stage (256)
    static constexpr int KC = 0, VC = CODEB, KP = 2 * CODEB, VP = 2 * CODEB + PARB;
    static constexpr int STAGE = 2 * (CODEB + PARB);
};

template <int D>
constexpr int attn_smem_bytes() {
    return kWarps * kRing * Geo<D>::STAGE + kWarps * kRing * 8 + kAlignSlack;
}

struct AttnParams {
    const uint16_t* q;   // BF16 [B][Hq][D]
    const uint8_t* kc;   // [B][Hkv][l_cap][D/2]
    const uint32_t* kp;  // [B][Hkv][l_cap][D/128]
    const uint8_t* vc;
    const uint32_t* vp;
    const int32_t* lens;  // [B]
    int hkv, G;
    int64_t l_cap;
    int max_len;
    float scale_log2;  // softmax scale * log2(e)
    int nsplit, spc;   // CTAs per (sequence, KV head), stages per CTA
    void* out;         // [B][Hq][D], BF16 or F32
    int out_f32;
    float* part_o;       // [B*Hkv][nsplit][G][D]  unnormalised outputs (nsplit > 1)
    float* part_ml;      // [B*Hkv][nsplit][G][2]  running max (log2 units) and sum
    unsigned* counters;  // [B*Hkv], zero between calls (nsplit > 1)
    int* status;
};

// f16x2 arithmetic on plain 32-bit registers (no __half2 round trips).
__device__ __forceinline__ uint32_t hadd2_u(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t hfma2_u(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
// (FP16(lo), FP16(hi)) packed, lo in bits 0..15.
__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}
// 2^x by the hardware approximation (relative error about 2^-22; -inf -> 0).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// 2^e for -126 <= e <= 127, exactly.
__device__ __forceinline__ float pow2i(int e) { return __int_as_float((e + 127) << 23); }

// The codes at bits 0..3 and 16..19 of w as the FP16 pair (c_lo - 8, c_hi - 8):
// 0x6400 | c is 1024 + c, exact; adding -1032 is exact.
__device__ __forceinline__ uint32_t dq_lo(uint32_t w) {
    return hadd2_u((w & 0x000F000Fu) | 0x64006400u, 0xE408E408u);
}
// The codes at bits 4..7 and 20..23: 0x6400 | 16 c is 1024 + 16 c; times 1/16
// minus 72 gives c - 8, exactly.
__device__ __forceinline__ uint32_t dq_hi(uint32_t w) {
    return hfma2_u((w & 0x00F000F0u) | 0x64006400u, 0x2C002C00u, 0xD480D480u);
}

__device__ __forceinline__ uint32_t movmatrix_t(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
}

__device__ __forceinline__ float f16lo(uint32_t w) { return __half2float(__ushort_as_half((uint16_t)(w & 0xFFFFu))); }
__device__ __forceinline__ float f16hi(uint32_t w) { return __half2float(__ushort_as_half((uint16_t)(w >> 16))); }

template <int D>
__global__ void __launch_bounds__(kWarps * 32, 1) attn_kernel(const AttnParams p) {
    using Gm = Geo<D>;
    constexpr int NG = Gm::NG, MT = Gm::MT, TS = Gm::TS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = ptx::align_smem<128>(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kWarps * kRing * Gm::STAGE);
    __shared__ int s_last;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int bh = blockIdx.y, c = blockIdx.x;
    const int b = bh / p.hkv, kvh = bh - b * p.hkv;
    uint8_t* ring = smem + warp * kRing * Gm::STAGE;
    uint64_t* full = bars + warp * kRing;
    if (lane == 0) {
        for (int i = 0; i < kRing; ++i) ptx::mbar_init(&full[i], 1);
        ptx::fence_barrier_init();
    }
    __syncwarp();
    ptx::pdl_launch_dependents();
    ptx::pdl_wait();  // q, lens and the cache may come from the kernels before

    int len = p.lens[b];
    if (len < 0 || len > p.max_len) {
        if (threadIdx.x == 0 && c == 0 && kvh == 0) record_status(p.status, BQ_ERR_SHAPE);
        len = min(max(len, 0), p.max_len);
    }
    const int ns = (len + TS - 1) / TS;
    const int s0 = c * p.spc + warp;
    const int s1 = min((c + 1) * p.spc, ns);
    const int nmy = s1 > s0 ? (s1 - s0 + kWarps - 1) / kWarps : 0;
    const int64_t tok_base = (int64_t)bh * p.l_cap;
    const uint8_t* kc = p.kc + tok_base * Gm::ROWB;
    const uint8_t* vc = p.vc + tok_base * Gm::ROWB;
    const uint32_t* kp = p.kp + tok_base * NG;
    const uint32_t* vp = p.vp + tok_base * NG;
    auto issue = [&](int i) {  // lane 0 only
        const int64_t tok = (int64_t)(s0 + kWarps * i) * TS;
        uint8_t* dst = ring + (i % kRing) * Gm::STAGE;
        uint64_t* bar = &full[i % kRing];
        ptx::mbar_arrive_expect_tx(bar, Gm::STAGE);
        ptx::bulk_load(dst + Gm::KC, kc + tok * Gm::ROWB, Gm::CODEB, bar);
        ptx::bulk_load(dst + Gm::VC, vc + tok * Gm::ROWB, Gm::CODEB, bar);
        ptx::bulk_load(dst + Gm::KP, kp + tok * NG, Gm::PARB, bar);
        ptx::bulk_load(dst + Gm::VP, vp + tok * NG, Gm::PARB, bar);
    };
    if (lane == 0)
        for (int i = 0; i < min(kRing, nmy); ++i) issue(i);

    // ---- query head g of this KV group, as int8 digit planes ----------------
    // Thread (g, t) holds dims 128 grp + 32 t + [0, 32) of head g.  Each value
    // becomes the integer q22 = rint(q 2^e) (the head's largest |q| in
    // [2^20, 2^21): exact for BF16 values within 2^-13 of it, else rounded by at
    // most 2^-21 of it), split into balanced base-256 digits d0, d1 in
    // [-128, 127] and d2 in [-33, 33] with q22 = 65536 d2 + 256 d1 + d0, one MMA
    // B operand per digit plane.  K-step u of group grp reads word u of the
    // thread's K codes: its even nibbles (dims 8u + 0, 2, 4, 6) fill k-slots
    // 4t .. 4t+3 (b0), its odd nibbles k-slots 4t+16 .. 4t+19 (b1).
    uint32_t qb[NG][4][3][2];
    float ch[2], dh[2][NG];
    {
        const bool hv = g < p.G;
        const uint16_t* qh = p.q + ((int64_t)bh * p.G + (hv ? g : 0)) * D;
        float v[NG][32];
        float mx = 0.f;
#pragma unroll
        for (int grp = 0; grp < NG; ++grp)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint4 raw = make_uint4(0u, 0u, 0u, 0u);
                if (hv) raw = __ldg(reinterpret_cast<const uint4*>(qh + 128 * grp + 32 * t + 8 * i));
                const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    v[grp][8 * i + 2 * e] = bf16_lo(w[e]);
                    v[grp][8 * i + 2 * e + 1] = bf16_hi(w[e]);
                    mx = fmaxf(mx, fmaxf(fabsf(v[grp][8 * i + 2 * e]), fabsf(v[grp][8 * i + 2 * e + 1])));
                }
            }
        mx = fmaxf(mx, __shfl_xor_sync(~0u, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(~0u, mx, 2));
        // (a head whose largest |q| is below 2^-106 keeps the factor 2^126)
        const int ex = mx > 0.f ? min(20 - ilogbf(mx), 126) : 0;
        const float fx = pow2i(ex);
        int sum[NG];
#pragma unroll
        for (int grp = 0; grp < NG; ++grp) {
            int qi[32];
            sum[grp] = 0;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                qi[i] = __float2int_rn(v[grp][i] * fx);
                sum[grp] += qi[i];
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                uint32_t b[2][3] = {{0u, 0u, 0u}, {0u, 0u, 0u}};
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int odd = 0; odd < 2; ++odd) {
                        const int a = qi[8 * u + 2 * i + odd];
                        const int d0 = ((a + 128) & 255) - 128;
                        const int r = (a - d0) >> 8;
                        const int d1 = ((r + 128) & 255) - 128;
                        const int d2 = (r - d1) >> 8;
                        b[odd][0] |= (uint32_t)(d0 & 255) << (8 * i);
                        b[odd][1] |= (uint32_t)(d1 & 255) << (8 * i);
                        b[odd][2] |= (uint32_t)(d2 & 255) << (8 * i);
                    }
#pragma unroll
                for (int j = 0; j < 3; ++j) {
                    qb[grp][u][j][0] = b[0][j];
                    qb[grp][u][j][1] = b[1][j];
                }
            }
            sum[grp] += __shfl_xor_sync(~0u, sum[grp], 1);
            sum[grp] += __shfl_xor_sync(~0u, sum[grp], 2);
        }
        // per-head constants of the score epilogue, for the heads 2t, 2t+1 this
        // thread's accumulator columns hold (head g' lives in lanes 4 g')
        const float cg = p.scale_log2 * pow2i(-ex);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            ch[j] = __shfl_sync(~0u, cg, 4 * (2 * t + j));
#pragma unroll
            for (int grp = 0; grp < NG; ++grp)
                dh[j][grp] = __shfl_sync(~0u, cg * (float)sum[grp], 4 * (2 * t + j));
        }
    }

    // ---- stream the context ------------------------------------------------
    float o[NG][8][4];
#pragma unroll
    for (int grp = 0; grp < NG; ++grp)
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) o[grp][i][e] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f}, z_run[NG][2];
#pragma unroll
    for (int grp = 0; grp < NG; ++grp) z_run[grp][0] = z_run[grp][1] = 0.f;
    int sig = kNoSigma;

    int done = 0;
    bool alive = true;
    for (int i = 0; i < nmy; ++i) {
        const int slot = i % kRing;
        const bool ok = ptx::mbar_wait_bounded(&full[slot], (uint32_t)((i / kRing) & 1), kWaitPolls);
        if (!__all_sync(~0u, ok)) {
            if (lane == 0) record_status(p.status, BQ_ERR_TIMEOUT);
            alive = false;
            break;
        }
        const uint8_t* sb = ring + slot * Gm::STAGE;
        const int tok0 = (s0 + kWarps * i) * TS;

        float sc[MT][4];
        float sv[MT][2][NG], wv[MT][2][NG];
        float smax = 0.f;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int r0 = mt * 16 + g, r1 = r0 + 8;
            const bool v0 = tok0 + r0 < len, v1 = tok0 + r1 < len;
            // S = sum_d q22_d c_d per (token row, head column), exact: three
            // int8 digit planes, one u8 x s8 MMA each per 32 dims
            float S[NG][4];
#pragma unroll
            for (int grp = 0; grp < NG; ++grp) {
                int acc[3][4];
#pragma unroll
                for (int j = 0; j < 3; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0;
                const uint4 k0 = *reinterpret_cast<const uint4*>(sb + Gm::KC + r0 * Gm::ROWB + 64 * grp + 16 * t);
                const uint4 k1 = *reinterpret_cast<const uint4*>(sb + Gm::KC + r1 * Gm::ROWB + 64 * grp + 16 * t);
                const uint32_t w0[4] = {k0.x, k0.y, k0.z, k0.w}, w1[4] = {k1.x, k1.y, k1.z, k1.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const uint32_t l0 = w0[u] & 0x0F0F0F0Fu, h0 = (w0[u] >> 4) & 0x0F0F0F0Fu;
                    const uint32_t l1 = w1[u] & 0x0F0F0F0Fu, h1 = (w1[u] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
                    for (int j = 0; j < 3; ++j)
                        ptx::mma_u8s8(acc[j], l0, l1, h0, h1, qb[grp][u][j][0], qb[grp][u][j][1]);
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    // |acc[2]| <= 33 * 15 * 128 < 2^22: to float by the 1.5 * 2^23
                    // bias; 256 acc[1] + acc[0] fits int32 exactly
                    const float hi = __int_as_float(acc[2][e] + 0x4B400000) - 12582912.0f;
                    S[grp][e] = fmaf(hi, 65536.0f, (float)(acc[1][e] * 256 + acc[0][e]));
                }
            }
            float s00 = 0.f, s01 = 0.f, s10 = 0.f, s11 = 0.f;
#pragma unroll
            for (int grp = 0; grp < NG; ++grp) {
                const uint32_t pk0 = *reinterpret_cast<const uint32_t*>(sb + Gm::KP + (r0 * NG + grp) * 4);
                const uint32_t pk1 = *reinterpret_cast<const uint32_t*>(sb + Gm::KP + (r1 * NG + grp) * 4);
                // score = s sum q c + z sum q (K = s c + z), in log2 units
                const float sk0 = f16lo(pk0), zk0 = f16hi(pk0);
                const float sk1 = f16lo(pk1), zk1 = f16hi(pk1);
                s00 = fmaf(S[grp][0], sk0 * ch[0], fmaf(zk0, dh[0][grp], s00));
                s01 = fmaf(S[grp][1], sk0 * ch[1], fmaf(zk0, dh[1][grp], s01));
                s10 = fmaf(S[grp][2], sk1 * ch[0], fmaf(zk1, dh[0][grp], s10));
                s11 = fmaf(S[grp][3], sk1 * ch[1], fmaf(zk1, dh[1][grp], s11));
                const uint32_t pv0 = *reinterpret_cast<const uint32_t*>(sb + Gm::VP + (r0 * NG + grp) * 4);
                const uint32_t pv1 = *reinterpret_cast<const uint32_t*>(sb + Gm::VP + (r1 * NG + grp) * 4);
                // tokens past the end: weight 0 and no V parameters (their bytes
                // are whatever the cache holds there)
                sv[mt][0][grp] = v0 ? f16lo(pv0) : 0.f;
                sv[mt][1][grp] = v1 ? f16lo(pv1) : 0.f;
                wv[mt][0][grp] = v0 ? fmaf(8.f, f16lo(pv0), f16hi(pv0)) : 0.f;
                wv[mt][1][grp] = v1 ? fmaf(8.f, f16lo(pv1), f16hi(pv1)) : 0.f;
                smax = fmaxf(smax, fmaxf(sv[mt][0][grp], sv[mt][1][grp]));
            }
            sc[mt][0] = v0 ? s00 : -INFINITY;
            sc[mt][1] = v0 ? s01 : -INFINITY;
            sc[mt][2] = v1 ? s10 : -INFINITY;
            sc[mt][3] = v1 ? s11 : -INFINITY;
        }

        // stage maxima (per head column over the 16 g rows) and the rescale
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            mx0 = fmaxf(mx0, fmaxf(sc[mt][0], sc[mt][2]));
            mx1 = fmaxf(mx1, fmaxf(sc[mt][1], sc[mt][3]));
        }
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(~0u, mx0, off));
            mx1 = fmaxf(mx1, __shfl_xor_sync(~0u, mx1, off));
            smax = fmaxf(smax, __shfl_xor_sync(~0u, smax, off));
        }
        smax = fmaxf(smax, __shfl_xor_sync(~0u, smax, 1));
        smax = fmaxf(smax, __shfl_xor_sync(~0u, smax, 2));
        const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
        const int sig_new = smax > 0.f ? min(sig, 14 - ilogbf(smax)) : sig;
        const float fl0 = (mn0 == -INFINITY) ? 1.f : ex2(m_run[0] - mn0);
        const float fl1 = (mn1 == -INFINITY) ? 1.f : ex2(m_run[1] - mn1);
        const float fs = pow2i(sig_new - sig);
        const float fo0 = fl0 * fs, fo1 = fl1 * fs;
        if (__any_sync(~0u, fo0 != 1.f || fo1 != 1.f)) {
#pragma unroll
            for (int grp = 0; grp < NG; ++grp)
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    o[grp][j][0] *= fo0;
                    o[grp][j][1] *= fo1;
                    o[grp][j][2] *= fo0;
                    o[grp][j][3] *= fo1;
                }
        }
        l_run[0] *= fl0;
        l_run[1] *= fl1;
#pragma unroll
        for (int grp = 0; grp < NG; ++grp) {
            z_run[grp][0] *= fl0;
            z_run[grp][1] *= fl1;
        }
        m_run[0] = mn0;
        m_run[1] = mn1;
        sig = sig_new;
        const float mref0 = mn0 == -INFINITY ? 0.f : mn0, mref1 = mn1 == -INFINITY ? 0.f : mn1;
        const float pscale = pow2i(sig);

        // P V
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const float p00 = ex2(sc[mt][0] - mref0), p01 = ex2(sc[mt][1] - mref1);
            const float p10 = ex2(sc[mt][2] - mref0), p11 = ex2(sc[mt][3] - mref1);
            l_run[0] += p00 + p10;
            l_run[1] += p01 + p11;
            const uint8_t* vrow = sb + Gm::VC + mt * 16 * Gm::ROWB + 8 * g;
#pragma unroll
            for (int grp = 0; grp < NG; ++grp) {
                z_run[grp][0] = fmaf(p00, wv[mt][0][grp], fmaf(p10, wv[mt][1][grp], z_run[grp][0]));
                z_run[grp][1] = fmaf(p01, wv[mt][0][grp], fmaf(p11, wv[mt][1][grp], z_run[grp][1]));
                const float f0 = sv[mt][0][grp] * pscale, f1 = sv[mt][1][grp] * pscale;
                // P'' of rows g / g+8 (tokens) and columns 2t, 2t+1 (heads),
                // transposed to the B fragment: (tokens 2t, 2t+1 | 2t+8, 2t+9; head g)
                const uint32_t b0 = movmatrix_t(pack_half2(p00 * f0, p01 * f0));
                const uint32_t b1 = movmatrix_t(pack_half2(p10 * f1, p11 * f1));
                const uint8_t* vg = vrow + 64 * grp;
                const uint2 va = *reinterpret_cast<const uint2*>(vg + (2 * t) * Gm::ROWB);
                const uint2 vb = *reinterpret_cast<const uint2*>(vg + (2 * t + 1) * Gm::ROWB);
                const uint2 vcw = *reinterpret_cast<const uint2*>(vg + (2 * t + 8) * Gm::ROWB);
                const uint2 vd = *reinterpret_cast<const uint2*>(vg + (2 * t + 9) * Gm::ROWB);
                const uint32_t wa[2] = {va.x, va.y}, wb[2] = {vb.x, vb.y}, wc[2] = {vcw.x, vcw.y},
                               wd[2] = {vd.x, vd.y};
#pragma unroll
                for (int w = 0; w < 2; ++w)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        // dims 16 g + 8 w + 4 hh + n of the group, tokens (2t | 2t+1)
                        // in X and (2t+8 | 2t+9) in Y
                        const uint32_t sel = hh ? 0x7632u : 0x5410u;
                        const uint32_t X = __byte_perm(wa[w], wb[w], sel);
                        const uint32_t Y = __byte_perm(wc[w], wd[w], sel);
                        const int i0 = 4 * w + 2 * hh;
                        ptx::mma_f16_16816(o[grp][i0], dq_lo(X), dq_hi(X), dq_lo(Y), dq_hi(Y), b0, b1);
                        ptx::mma_f16_16816(o[grp][i0 + 1], dq_lo(X >> 8), dq_hi(X >> 8), dq_lo(Y >> 8),
                                           dq_hi(Y >> 8), b0, b1);
                    }
            }
        }
        done = i + 1;
        __syncwarp();
        if (lane == 0 && i + kRing < nmy) issue(i + kRing);
    }
    if (!alive) {
        // copies still in flight land before the CTA exits (bounded)
        for (int k = done; k < min(nmy, done + kRing); ++k)
            ptx::mbar_wait_bounded(&full[k % kRing], (uint32_t)((k / kRing) & 1), kWaitPolls);
    }

    // ---- per-warp totals ---------------------------------------------------
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        l_run[0] += __shfl_xor_sync(~0u, l_run[0], off);
        l_run[1] += __shfl_xor_sync(~0u, l_run[1], off);
#pragma unroll
        for (int grp = 0; grp < NG; ++grp) {
            z_run[grp][0] += __shfl_xor_sync(~0u, z_run[grp][0], off);
            z_run[grp][1] += __shfl_xor_sync(~0u, z_run[grp][1], off);
        }
    }
    __syncthreads();  // every warp is done with its ring: reuse it for the merge
    float* mo = reinterpret_cast<float*>(smem);          // [kWarps][8][D]
    float* mm = mo + kWarps * kMaxHeads * D;              // [kWarps][8]
    float* ml = mm + kWarps * kMaxHeads;                  // [kWarps][8]
    float* wgt = ml + kWarps * kMaxHeads;                 // [nsplit][8], then [8] totals
    const float inv = pow2i(-sig);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int h = 2 * t + j;
        if (h < p.G) {
            float* dst = mo + (warp * kMaxHeads + h) * D;
#pragma unroll
            for (int grp = 0; grp < NG; ++grp)
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int d0 = 128 * grp + 16 * g + 2 * i;
                    dst[d0] = fmaf(o[grp][i][j], inv, z_run[grp][j]);
                    dst[d0 + 1] = fmaf(o[grp][i][2 + j], inv, z_run[grp][j]);
                }
            if (g == 0) {
                mm[warp * kMaxHeads + h] = m_run[j];
                ml[warp * kMaxHeads + h] = l_run[j];
            }
        }
    }
    __syncthreads();

    // ---- merge the warps (in warp order) -----------------------------------
    const int nout = p.G * D;
    for (int idx = threadIdx.x; idx < nout; idx += blockDim.x) {
        const int h = idx / D, d = idx - h * D;
        float M = -INFINITY;
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mm[w * kMaxHeads + h]);
        float O = 0.f, L = 0.f;
        if (M != -INFINITY)
            for (int w = 0; w < kWarps; ++w) {
                const float a = exp2f(mm[w * kMaxHeads + h] - M);
                O = fmaf(a, mo[(w * kMaxHeads + h) * D + d], O);
                L = fmaf(a, ml[w * kMaxHeads + h], L);
            }
        const int64_t oi = ((int64_t)bh * p.G + h) * D + d;
        if (p.nsplit == 1) {
            const float r = L > 0.f ? O / L : 0.f;
            if (p.out_f32)
                static_cast<float*>(p.out)[oi] = r;
            else
                static_cast<uint16_t*>(p.out)[oi] = float_to_bf16_bits(r);
        } else {
            const int64_t slot = ((int64_t)bh * p.nsplit + c) * p.G + h;
            p.part_o[slot * D + d] = O;
            if (d == 0) {
                p.part_ml[2 * slot] = M;
                p.part_ml[2 * slot + 1] = L;
            }
        }
    }
    if (p.nsplit == 1) return;

    // ---- the last CTA of this (sequence, KV head) merges the splits ---------
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(&p.counters[bh], 1u) == (unsigned)(p.nsplit - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // every split's (max, sum) into shared memory, all loads in flight at once
    const int nsg = p.nsplit * p.G;
    const float* pml = p.part_ml + (int64_t)bh * nsg * 2;
    float* sw = wgt;                 // [nsplit * G] maxima, then weights
    float* sl = wgt + nsg;           // [nsplit * G] sums
    float* tot = sl + nsg;           // [G] totals
    for (int i = threadIdx.x; i < nsg; i += blockDim.x) {
        const float2 v = __ldcg(reinterpret_cast<const float2*>(pml) + i);
        sw[i] = v.x;
        sl[i] = v.y;
    }
    __syncthreads();
    if (threadIdx.x < p.G) {
        const int h = threadIdx.x;
        float M = -INFINITY;
        for (int cc = 0; cc < p.nsplit; ++cc) M = fmaxf(M, sw[cc * p.G + h]);
        float L = 0.f;
        for (int cc = 0; cc < p.nsplit; ++cc) {
            const float a = M == -INFINITY ? 0.f : exp2f(sw[cc * p.G + h] - M);
            sw[cc * p.G + h] = a;
            L = fmaf(a, sl[cc * p.G + h], L);
        }
        tot[h] = L;
    }
    __syncthreads();
    // outputs four at a time; the split loop is unrolled so that its loads are
    // issued together (the sum is still taken in split order)
    const float* po = p.part_o + (int64_t)bh * nsg * D;
    const int nq = p.G * (D / 4);
    for (int idx = threadIdx.x; idx < nq; idx += blockDim.x) {
        const int h = idx / (D / 4), d = 4 * (idx - h * (D / 4));
        float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
        for (int cc = 0; cc < p.nsplit; ++cc) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(po + ((int64_t)cc * p.G + h) * D + d));
            const float a = sw[cc * p.G + h];
            O.x = fmaf(a, v.x, O.x);
            O.y = fmaf(a, v.y, O.y);
            O.z = fmaf(a, v.z, O.z);
            O.w = fmaf(a, v.w, O.w);
        }
        const float L = tot[h];
        const float r[4] = {L > 0.f ? O.x / L : 0.f, L > 0.f ? O.y / L : 0.f, L > 0.f ? O.z / L : 0.f,
                            L > 0.f ? O.w / L : 0.f};
        const int64_t oi = ((int64_t)bh * p.G + h) * D + d;
        if (p.out_f32) {
            *reinterpret_cast<float4*>(static_cast<float*>(p.out) + oi) = make_float4(r[0], r[1], r[2], r[3]);
        } else {
            const uint32_t lo = float_to_bf16_bits(r[0]) | ((uint32_t)float_to_bf16_bits(r[1]) << 16);
            const uint32_t hi = float_to_bf16_bits(r[2]) | ((uint32_t)float_to_bf16_bits(r[3]) << 16);
            *reinterpret_cast<uint2*>(static_cast<uint16_t*>(p.out) + oi) = make_uint2(lo, hi);
        }
    }
    if (threadIdx.x == 0) p.counters[bh] = 0u;  // left zero for the next call
}

// ---- quantiser ---------------------------------------------------------------
// One warp per 128-value group; lane l holds values 4l .. 4l+3.
__device__ __forceinline__ void quant_group(const uint16_t* src, uint8_t* codes, uint32_t* param, int lane,
                                            int* status) {
    const uint2 raw = __ldg(reinterpret_cast<const uint2*>(src) + lane);
    const float v[4] = {bf16_lo(raw.x), bf16_hi(raw.x), bf16_lo(raw.y), bf16_hi(raw.y)};
    const bool fin = isfinite(v[0]) && isfinite(v[1]) && isfinite(v[2]) && isfinite(v[3]);
    uint16_t out = 0;
    uint32_t par = 0;
    if (!__all_sync(~0u, fin)) {
        if (lane == 0) record_status(status, BQ_ERR_NONFINITE);
    } else {
        float lo = fminf(fminf(v[0], v[1]), fminf(v[2], v[3])), hi = fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3]));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(~0u, lo, off));
            hi = fmaxf(hi, __shfl_xor_sync(~0u, hi, off));
        }
        const __half sh = __double2half(((double)hi - (double)lo) / 15.0);
        const __half zh = __double2half((double)lo);
        const double s = (double)__half2float(sh), z = (double)__half2float(zh);
        if (!isfinite(s) || !isfinite(z)) {
            if (lane == 0) record_status(status, BQ_ERR_SCALE_RANGE);
        } else {
            uint32_t cc[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const double q = s > 0.0 ? rint(((double)v[i] - z) / s) : 0.0;
                cc[i] = (uint32_t)fmin(fmax(q, 0.0), 15.0);
            }
            out = (uint16_t)(cc[0] | (cc[1] << 4) | (cc[2] << 8) | (cc[3] << 12));
            par = (uint32_t)__half_as_ushort(sh) | ((uint32_t)__half_as_ushort(zh) << 16);
        }
    }
    reinterpret_cast<uint16_t*>(codes)[lane] = out;
    if (lane == 0) *param = par;
}

constexpr int kQuantWarps = 8;

__global__ void __launch_bounds__(kQuantWarps * 32) quantize_kernel(const uint16_t* __restrict__ x, int64_t groups,
                                                                    uint8_t* __restrict__ codes,
                                                                    uint32_t* __restrict__ params, int* status) {
    ptx::pdl_launch_dependents();
    ptx::pdl_wait();
    const int64_t gi = (int64_t)blockIdx.x * kQuantWarps + (threadIdx.x >> 5);
    if (gi >= groups) return;
    quant_group(x + gi * 128, codes + gi * 64, params + gi, threadIdx.x & 31, status);
}

// Warp per (sequence, KV head, K or V, group): the new token's vector goes to
// row pos[b] of its cache.
__global__ void __launch_bounds__(kQuantWarps * 32)
    append_kernel(const uint16_t* __restrict__ k, const uint16_t* __restrict__ v, int batch, int hkv, int ng,
                  const int32_t* __restrict__ pos, int64_t l_cap, uint8_t* kc, uint32_t* kp, uint8_t* vc,
                  uint32_t* vp, int* status) {
    ptx::pdl_launch_dependents();
    ptx::pdl_wait();
    const int64_t gi = (int64_t)blockIdx.x * kQuantWarps + (threadIdx.x >> 5);
    const int64_t per_kv = 2LL * ng;
    if (gi >= (int64_t)batch * hkv * per_kv) return;
    const int64_t bh = gi / per_kv;
    const int r = (int)(gi - bh * per_kv);
    const int isv = r >= ng, grp = isv ? r - ng : r;
    const int b = (int)(bh / hkv);
    const int32_t ps = __ldg(pos + b);
    if (ps < 0 || (int64_t)ps >= l_cap) {
        if ((threadIdx.x & 31) == 0) record_status(status, BQ_ERR_SHAPE);
        return;
    }
    const int d = 128 * ng;
    const uint16_t* src = (isv ? v : k) + bh * d + 128 * grp;
    const int64_t row = bh * l_cap + ps;
    uint8_t* codes = (isv ? vc : kc) + row * (d / 2) + 64 * grp;
    uint32_t* par = (isv ? vp : kp) + row * ng + grp;
    quant_group(src, codes, par, threadIdx.x & 31, status);
}

// ---- host side -----------------------------------------------------------------
struct Plan {
    int nsplit = 1, spc = 0;
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool attn_shape_ok(int batch, int hq, int hkv, int d, int64_t l_cap, int64_t max_len) {
    if (d != 128 && d != 256) return false;
    if (batch < 0 || hkv < 1 || hq < 1 || hq % hkv != 0 || hq / hkv > kMaxHeads) return false;
    if ((int64_t)batch * hkv > 65535) return false;
    if (l_cap < 0 || l_cap % 64 != 0 || max_len < 0 || max_len > l_cap || max_len > (1LL << 30)) return false;
    return true;
}

Plan make_plan(int batch, int hkv, int d, int64_t max_len) {
    Plan pl;
    const int ts = 8192 / d;
    const int64_t ns = (max_len + ts - 1) / ts;
    if (ns == 0 || batch == 0) return pl;
    const int64_t units = (int64_t)batch * hkv;
    int64_t nsplit = std::max<int64_t>(1, sm_count() / units);
    nsplit = std::min<int64_t>(nsplit, (ns + kWarps - 1) / kWarps);
    nsplit = std::max<int64_t>(nsplit, 1);
    const int64_t spc = (ns + nsplit - 1) / nsplit;
    pl.spc = (int)spc;
    pl.nsplit = (int)((ns + spc - 1) / spc);
    return pl;
}

int64_t round256(int64_t b) { return (b + 255) / 256 * 256; }

int64_t workspace_bytes(const Plan& pl, int batch, int hq, int hkv, int d) {
    if (pl.nsplit <= 1) return 0;
    const int64_t units = (int64_t)batch * hkv;
    const int64_t slots = units * pl.nsplit * (int64_t)(hq / hkv);
    return round256(slots * d * 4) + round256(slots * 8) + round256(units * 4);
}

template <int D>
cudaError_t launch_attn(const AttnParams& p, int units, cudaStream_t s) {
    const int smem = attn_smem_bytes<D>();
    cudaError_t e = ensure_dynamic_smem((const void*)attn_kernel<D>, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.nsplit, (unsigned)units);
    cfg.blockDim = dim3(kWarps * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, attn_kernel<D>, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_pdl_1d(const void* func, int64_t warps, void** args, cudaStream_t s) {
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((warps + kQuantWarps - 1) / kQuantWarps));
    cfg.blockDim = dim3(kQuantWarps * 32);
    cfg.stream = s;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelExC(&cfg, func, args);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace
}  // namespace kv4
}  // namespace bq

using namespace bq;

extern "C" int64_t bq_kv4_codes_bytes(int64_t rows, int d) {
    if (rows < 0 || (d != 128 && d != 256)) return -1;
    return rows * d / 2;
}

extern "C" int64_t bq_kv4_params_bytes(int64_t rows, int d) {
    if (rows < 0 || (d != 128 && d != 256)) return -1;
    return rows * (d / 128) * 4;
}

extern "C" bq_status bq_kv4_quantize(const uint16_t* x, int64_t rows, int d, uint8_t* codes, uint32_t* params,
                                     void* stream) {
    if (rows < 0 || (d != 128 && d != 256) || rows > (1LL << 40) / d) return BQ_ERR_SHAPE;
    if (rows == 0) return BQ_OK;
    if (!x || !codes || !params) return BQ_ERR_NULL;
    if (!kv4::aligned16(x) || !kv4::aligned16(codes) || !kv4::aligned16(params)) return BQ_ERR_ALIGN;
    int* status = device_status_ptr();
    if (!status) return BQ_ERR_CUDA;
    int64_t groups = rows * (d / 128);
    void* args[] = {&x, &groups, &codes, &params, &status};
    const cudaError_t e = kv4::launch_pdl_1d((const void*)kv4::quantize_kernel, groups, args,
                                             static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

extern "C" bq_status bq_kv4_append(const uint16_t* k, const uint16_t* v, int batch, int hkv, int d,
                                   const int32_t* pos, int64_t l_cap, uint8_t* k_codes, uint32_t* k_params,
                                   uint8_t* v_codes, uint32_t* v_params, void* stream) {
    if (batch < 0 || hkv < 1 || (d != 128 && d != 256) || l_cap < 1 || l_cap % 64 != 0 ||
        (int64_t)batch * hkv > (1LL << 24))
        return BQ_ERR_SHAPE;
    if (batch == 0) return BQ_OK;
    if (!k || !v || !pos || !k_codes || !k_params || !v_codes || !v_params) return BQ_ERR_NULL;
    if (!kv4::aligned16(k) || !kv4::aligned16(v) || (reinterpret_cast<uintptr_t>(pos) & 3u) ||
        !kv4::aligned16(k_codes) || !kv4::aligned16(k_params) || !kv4::aligned16(v_codes) ||
        !kv4::aligned16(v_params))
        return BQ_ERR_ALIGN;
    int* status = device_status_ptr();
    if (!status) return BQ_ERR_CUDA;
    int ng = d / 128;
    const int64_t warps = (int64_t)batch * hkv * 2 * ng;
    void* args[] = {&k, &v, &batch, &hkv, &ng, &pos, &l_cap, &k_codes, &k_params, &v_codes, &v_params, &status};
    const cudaError_t e =
        kv4::launch_pdl_1d((const void*)kv4::append_kernel, warps, args, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

extern "C" int64_t bq_kv4_attention_workspace_bytes(int batch, int hq, int hkv, int d, int64_t l_cap,
                                                    int64_t max_len) {
    if (!kv4::attn_shape_ok(batch, hq, hkv, d, l_cap, max_len)) return -1;
    return kv4::workspace_bytes(kv4::make_plan(batch, hkv, d, max_len), batch, hq, hkv, d);
}

extern "C" bq_status bq_kv4_attention_decode(const uint16_t* q, const uint8_t* k_codes, const uint32_t* k_params,
                                             const uint8_t* v_codes, const uint32_t* v_params, const int32_t* lens,
                                             int batch, int hq, int hkv, int d, int64_t l_cap, int64_t max_len,
                                             float scale, void* out, int out_dtype, void* workspace,
                                             size_t workspace_bytes, void* stream) {
    if (!kv4::attn_shape_ok(batch, hq, hkv, d, l_cap, max_len)) return BQ_ERR_SHAPE;
    if (out_dtype != BQ_BF16 && out_dtype != BQ_F32) return BQ_ERR_FORMAT;
    if (!isfinite(scale)) return BQ_ERR_SHAPE;
    if (batch == 0) return BQ_OK;
    if (!q || !lens || !out || (l_cap > 0 && (!k_codes || !k_params || !v_codes || !v_params))) return BQ_ERR_NULL;
    if (!kv4::aligned16(q) || !kv4::aligned16(out) || (reinterpret_cast<uintptr_t>(lens) & 3u) ||
        (l_cap > 0 && (!kv4::aligned16(k_codes) || !kv4::aligned16(k_params) || !kv4::aligned16(v_codes) ||
                       !kv4::aligned16(v_params))))
        return BQ_ERR_ALIGN;
    const kv4::Plan pl = kv4::make_plan(batch, hkv, d, max_len);
    const int64_t need = kv4::workspace_bytes(pl, batch, hq, hkv, d);
    if (need > 0 && (!workspace || (int64_t)workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)))
        return BQ_ERR_WORKSPACE;
    int* status = device_status_ptr();
    if (!status) return BQ_ERR_CUDA;
    kv4::AttnParams p;
    p.q = q;
    p.kc = k_codes;
    p.kp = k_params;
    p.vc = v_codes;
    p.vp = v_params;
    p.lens = lens;
    p.hkv = hkv;
    p.G = hq / hkv;
    p.l_cap = l_cap;
    p.max_len = (int)max_len;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.nsplit = pl.nsplit;
    p.spc = pl.spc;
    p.out = out;
    p.out_f32 = out_dtype == BQ_F32;
    const int64_t units = (int64_t)batch * hkv;
    const int64_t slots = units * pl.nsplit * (int64_t)p.G;
    uint8_t* wsb = static_cast<uint8_t*>(workspace);
    p.part_o = need > 0 ? reinterpret_cast<float*>(wsb) : nullptr;
    p.part_ml = need > 0 ? reinterpret_cast<float*>(wsb + kv4::round256(slots * d * 4)) : nullptr;
    p.counters = need > 0 ? reinterpret_cast<unsigned*>(wsb + kv4::round256(slots * d * 4) + kv4::round256(slots * 8))
                          : nullptr;
    p.status = status;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const cudaError_t e = d == 128 ? kv4::launch_attn<128>(p, (int)units, s) : kv4::launch_attn<256>(p, (int)units, s);
    return e == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}
