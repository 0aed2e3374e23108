// C ABI entry points: argument validation on the host, dispatch to the
// kernels, device status words and their read-back.  Nothing here computes
// on the data path.
#include <mutex>

#include "bq_internal.cuh"

namespace bq {

namespace {

__device__ int g_device_status = 0;
__device__ unsigned long long g_pack_first_error = ~0ull;

std::mutex g_pack_mutex;

inline bool fmt_ok(int fmt) {
    return fmt == BQ_Q1G128 || fmt == BQ_T2G128 || fmt == BQ_T5P8G128 || fmt == BQ_A1G128;
}
inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

__global__ void wait_never_set_kernel(int64_t spin_limit, const volatile int* flag, int* status) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    for (int64_t i = 0; i < spin_limit; ++i) {
        if (*flag != 0) return;
        __nanosleep(32);
    }
    record_status(status, BQ_ERR_TIMEOUT);
}

__device__ int g_never_set_flag = 0;

bq_status validate_matrix(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k) {
    if (!fmt_ok(fmt)) return BQ_ERR_FORMAT;
    if (n < 0 || k < 0 || k % kGroup != 0) return BQ_ERR_SHAPE;
    if (n > 0 && k > 0) {
        if (!codes || !scales) return BQ_ERR_NULL;
        if (!aligned(codes, 16) || !aligned(scales, 16)) return BQ_ERR_ALIGN;
    }
    return BQ_OK;
}

bq_status pack_common(int fmt, const float* w, int64_t n, int64_t k, const uint16_t* scales_in,
                      uint8_t* codes, uint16_t* scales, void* stream) {
    if (!fmt_ok(fmt)) return BQ_ERR_FORMAT;
    if (n < 0 || k < 0 || k % kGroup != 0) return BQ_ERR_SHAPE;
    if (n == 0 || k == 0) return BQ_OK;
    if (!w || !codes || !scales) return BQ_ERR_NULL;
    if (!aligned(w, 16) || !aligned(codes, 16) || !aligned(scales, 16) ||
        (scales_in && !aligned(scales_in, 16)))
        return BQ_ERR_ALIGN;
    std::lock_guard<std::mutex> lock(g_pack_mutex);
    cudaStream_t s = as_stream(stream);
    const unsigned long long none = ~0ull;
    if (cudaMemcpyToSymbolAsync(g_pack_first_error, &none, sizeof(none), 0,
                                cudaMemcpyHostToDevice, s) != cudaSuccess)
        return BQ_ERR_CUDA;
    unsigned long long* first_ptr = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&first_ptr), g_pack_first_error) != cudaSuccess)
        return BQ_ERR_CUDA;
    if (launch_pack(fmt, w, n, k, scales_in, codes, scales, first_ptr, s) != cudaSuccess)
        return BQ_ERR_CUDA;
    unsigned long long first = 0;
    if (cudaMemcpyFromSymbolAsync(&first, g_pack_first_error, sizeof(first), 0,
                                  cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return BQ_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return BQ_ERR_CUDA;
    if (first != ~0ull) return static_cast<bq_status>(first & 0xFF);
    return BQ_OK;
}

}  // namespace

int* device_status_ptr() {
    int* p = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_device_status) != cudaSuccess) return nullptr;
    return p;
}

}  // namespace bq

namespace bq {
// Batch 5..16 takes the wide-batch kernel wherever it is eligible: measured
// on B200 (one launch per matrix, weights larger than L2) it is as fast as or
// faster than the row-owning kernel at batch 5..8 (binary 4096 x 4096 batch 5:
// 7.8 vs 9.1 us; 4096 x 12288: 15.2 vs 37.9 us) and than the tcgen05 GEMM at
// batch 9..16 (binary 4096 x 4096 batch 16: 15.1 vs 18.8 us; 24576 x 4096:
// 26.8 vs 62.7 us).
GemvPath gemv_path(int fmt, int64_t n, int64_t k, int batch) {
    // (the 5-trit format takes it from batch 9, where the alternative is the
    // GEMM; at batch 5..8 it keeps the row-owning kernel)
    if (batch >= (fmt == BQ_T5P8G128 ? 9 : 5) && gemv_wide_eligible(fmt, n, k, batch)) return GemvPath::Wide;
    if (gemv_rows_eligible(fmt, n, k, batch)) return GemvPath::Rows;
    if (gemv_tc_eligible(fmt, n, k, batch)) return GemvPath::SplitK;
    if (gemm_tc_eligible(fmt, n, k, batch)) return GemvPath::Gemm;
    return GemvPath::None;
}

int64_t gemv_workspace_bytes(int fmt, int64_t n, int64_t k, int batch) {
    switch (gemv_path(fmt, n, k, batch)) {
        case GemvPath::SplitK: return gemv_tc_workspace_bytes(fmt, n, k, batch);
        case GemvPath::Gemm: return gemm_tc_workspace_bytes(n, k, batch);
        default: return 0;
    }
}

cudaError_t launch_gemv(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                        const uint16_t* x, int batch, void* y, int y_dtype, void* workspace, cudaStream_t s) {
    switch (gemv_path(fmt, n, k, batch)) {
        case GemvPath::Rows: return launch_gemv_rows(fmt, codes, scales, n, k, x, batch, y, y_dtype, s);
        case GemvPath::Wide: return launch_gemv_wide(fmt, codes, scales, n, k, x, batch, y, y_dtype, s);
        case GemvPath::SplitK: return launch_gemv_tc(fmt, codes, scales, n, k, x, batch, y, y_dtype, workspace, s);
        case GemvPath::Gemm: return launch_gemm_tc(fmt, codes, scales, n, k, x, batch, y, y_dtype, workspace, s);
        default: return cudaErrorInvalidValue;
    }
}
}  // namespace bq

using namespace bq;

extern "C" {

int64_t bq_codes_bytes(int fmt, int64_t n, int64_t k) {
    if (!fmt_ok(fmt) || n < 0 || k < 0 || k % kGroup) return -1;
    if (fmt == BQ_Q1G128 || fmt == BQ_A1G128) return n * (k / 8);
    if (fmt == BQ_T2G128) return n * (k / 4);
    return n * (k / kGroup) * 26;
}

int64_t bq_scales_bytes(int64_t n, int64_t k) {
    if (n < 0 || k < 0 || k % kGroup) return -1;
    return n * (k / kGroup) * 2;
}

int64_t bq_group_params_bytes(int fmt, int64_t n, int64_t k) {
    if (!fmt_ok(fmt) || n < 0 || k < 0 || k % kGroup) return -1;
    return n * (k / kGroup) * (fmt == BQ_A1G128 ? 4 : 2);
}

double bq_effective_bits(int fmt) {
    if (!fmt_ok(fmt)) return -1.0;
    return 8.0 * (double)(bq_codes_bytes(fmt, 1, kGroup) + bq_group_params_bytes(fmt, 1, kGroup)) / (double)kGroup;
}

bq_status bq_pack_q1g128(const float* w, int64_t n, int64_t k, const uint16_t* scales_in,
                         uint8_t* codes, uint16_t* scales, void* stream) {
    return pack_common(BQ_Q1G128, w, n, k, scales_in, codes, scales, stream);
}
bq_status bq_pack_t2g128(const float* w, int64_t n, int64_t k, const uint16_t* scales_in,
                         uint8_t* codes, uint16_t* scales, void* stream) {
    return pack_common(BQ_T2G128, w, n, k, scales_in, codes, scales, stream);
}
bq_status bq_pack_t5p8(const float* w, int64_t n, int64_t k, const uint16_t* scales_in,
                       uint8_t* codes, uint16_t* scales, void* stream) {
    return pack_common(BQ_T5P8G128, w, n, k, scales_in, codes, scales, stream);
}
bq_status bq_pack_a1g128(const float* w, int64_t n, int64_t k, const uint16_t* params_in,
                         uint8_t* codes, uint16_t* params, void* stream) {
    return pack_common(BQ_A1G128, w, n, k, params_in, codes, params, stream);
}


int bq_gemv_launches(int fmt, int64_t n, int64_t k, int batch) {
    if (!fmt_ok(fmt) || n < 0 || k < 0 || k % kGroup || batch < 1 || batch > BQ_MAX_BATCH) return -1;
    if (n == 0) return 0;
    if (k == 0) return 0;  // the output is cleared with a memset, no kernel
    switch (gemv_path(fmt, n, k, batch)) {
        case GemvPath::Rows: return 1;
        case GemvPath::Wide: return 1;
        case GemvPath::SplitK: return 2;  // activation prep + split-K kernel
        case GemvPath::Gemm: return gemm_tc_launches(n, k, batch);
        default: return -1;  // no kernel takes the shape (bq_gemv returns BQ_ERR_SHAPE)
    }
}

int64_t bq_gemv_workspace_bytes(int fmt, int64_t n, int64_t k, int batch) {
    if (!fmt_ok(fmt) || n < 0 || k < 0 || k % kGroup || batch < 1 || batch > BQ_MAX_BATCH) return -1;
    if (n == 0 || k == 0) return 0;
    if (gemv_path(fmt, n, k, batch) == GemvPath::None) return -1;
    return gemv_workspace_bytes(fmt, n, k, batch);
}

bq_status bq_gemv(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                  const uint16_t* x, int batch, void* y, int y_dtype, void* workspace,
                  size_t workspace_bytes, void* stream) {
    bq_status st = validate_matrix(fmt, codes, scales, n, k);
    if (st != BQ_OK) return st;
    if (batch < 1 || batch > BQ_MAX_BATCH) return BQ_ERR_SHAPE;
    if (y_dtype != BQ_BF16 && y_dtype != BQ_F32) return BQ_ERR_FORMAT;
    if (n == 0) return BQ_OK;
    if (!y || (k > 0 && !x)) return BQ_ERR_NULL;
    if (!aligned(y, 16) || (x && !aligned(x, 16))) return BQ_ERR_ALIGN;
    const int64_t need = bq_gemv_workspace_bytes(fmt, n, k, batch);
    if (need < 0) return BQ_ERR_SHAPE;
    if (need > 0 && (!workspace || workspace_bytes < (size_t)need)) return BQ_ERR_WORKSPACE;
    if (workspace && !aligned(workspace, 256)) return BQ_ERR_ALIGN;
    if (k == 0) {
        const size_t bytes = (size_t)batch * n * (y_dtype == BQ_F32 ? 4 : 2);
        return cudaMemsetAsync(y, 0, bytes, as_stream(stream)) == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
    }
    const cudaError_t e = launch_gemv(fmt, codes, scales, n, k, x, batch, y, y_dtype, workspace, as_stream(stream));
    return e == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

// Prefill dispatch: up to 4 tokens run the tensor-core GEMV paths, and 5..16
// tokens the wide-batch GEMV where it takes the shape (the weight stream
// dominates; the result is bit-identical with bq_gemv); more tokens run the
// tcgen05 GEMM.  A shape neither takes (K > 2^28, N >= 2^31) is
// rejected with BQ_ERR_SHAPE.
static bool gemm_uses_gemv(int fmt, int64_t n, int64_t k, int64_t t) {
    if (t > BQ_MAX_BATCH) return false;
    const GemvPath p = gemv_path(fmt, n, k, (int)t);
    return (t <= 4 && (p == GemvPath::Rows || p == GemvPath::SplitK)) || p == GemvPath::Wide;
}

int64_t bq_gemm_workspace_bytes(int fmt, int64_t n, int64_t k, int64_t t) {
    if (!fmt_ok(fmt) || fmt == BQ_A1G128 || n < 0 || k < 0 || k % kGroup || t < 0) return -1;
    if (t == 0 || n == 0 || k == 0) return 0;
    if (gemm_uses_gemv(fmt, n, k, t)) return gemv_workspace_bytes(fmt, n, k, (int)t);
    if (gemm_tc_eligible(fmt, n, k, t)) return gemm_tc_workspace_bytes(n, k, t);
    return -1;
}

int bq_gemm_launches(int fmt, int64_t n, int64_t k, int64_t t) {
    if (!fmt_ok(fmt) || fmt == BQ_A1G128 || n < 0 || k < 0 || k % kGroup || t < 0) return -1;
    if (t == 0 || n == 0 || k == 0) return 0;
    if (gemm_uses_gemv(fmt, n, k, t)) return bq_gemv_launches(fmt, n, k, (int)t);
    if (gemm_tc_eligible(fmt, n, k, t)) return gemm_tc_launches(n, k, t);
    return -1;
}

bq_status bq_gemm(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                  const uint16_t* x, int64_t t, uint16_t* y, void* workspace, size_t workspace_bytes,
                  void* stream) {
    if (fmt == BQ_A1G128) return BQ_ERR_FORMAT;  // the prefill GEMM does not take the affine variant
    bq_status st = validate_matrix(fmt, codes, scales, n, k);
    if (st != BQ_OK) return st;
    if (t < 0) return BQ_ERR_SHAPE;
    if (n == 0 || t == 0) return BQ_OK;
    if (!y || (k > 0 && !x)) return BQ_ERR_NULL;
    if (!aligned(y, 16) || (x && !aligned(x, 16))) return BQ_ERR_ALIGN;
    const int64_t need = bq_gemm_workspace_bytes(fmt, n, k, t);
    if (need < 0) return BQ_ERR_SHAPE;
    if (need > 0 && (!workspace || workspace_bytes < (size_t)need)) return BQ_ERR_WORKSPACE;
    if (workspace && !aligned(workspace, 256)) return BQ_ERR_ALIGN;
    cudaStream_t s = as_stream(stream);
    if (k == 0)
        return cudaMemsetAsync(y, 0, (size_t)t * n * 2, s) == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
    cudaError_t e = cudaSuccess;
    if (gemm_uses_gemv(fmt, n, k, t))
        e = launch_gemv(fmt, codes, scales, n, k, x, (int)t, y, BQ_BF16, workspace, s);
    else
        e = launch_gemm_tc(fmt, codes, scales, n, k, x, t, y, BQ_BF16, workspace, s);
    return e == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

bq_status bq_embed_rows(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                        const int32_t* ids, int64_t count, uint16_t* out, void* stream) {
    bq_status st = validate_matrix(fmt, codes, scales, n, k);
    if (st != BQ_OK) return st;
    if (count < 0 || count > (int64_t)INT32_MAX * 8) return BQ_ERR_SHAPE;
    if (count == 0 || k == 0) return BQ_OK;
    if (!ids || !out) return BQ_ERR_NULL;
    if (!aligned(ids, 4) || !aligned(out, 16)) return BQ_ERR_ALIGN;
    const cudaError_t e = launch_embed_rows(fmt, codes, scales, n, k, ids, count, out, as_stream(stream));
    return e == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

int64_t bq_gemv_chain_workspace_bytes(void) { return 256; }

bq_status bq_gemv_chain(int fmt, const bq_chain_step* steps, int nsteps, int batch,
                        void* workspace, size_t workspace_bytes, void* stream) {
    if (!fmt_ok(fmt) || fmt == BQ_A1G128) return BQ_ERR_FORMAT;
    if (!steps) return BQ_ERR_NULL;
    if (nsteps < 1 || nsteps > BQ_MAX_CHAIN_STEPS || batch < 1 || batch > BQ_MAX_BATCH) return BQ_ERR_SHAPE;
    for (int i = 0; i < nsteps; ++i) {
        const bq_chain_step& st = steps[i];
        const bq_status v = validate_matrix(fmt, st.codes, st.scales, st.n, st.k);
        if (v != BQ_OK) return v;
        if (st.swiglu != 0 && st.swiglu != 1) return BQ_ERR_FORMAT;
        if (!st.swiglu && st.y_dtype != BQ_BF16 && st.y_dtype != BQ_F32) return BQ_ERR_FORMAT;
        if (st.n == 0 || st.k == 0) return BQ_ERR_SHAPE;
        if (!st.x || !st.y) return BQ_ERR_NULL;
        if (!aligned(st.x, 16) || !aligned(st.y, 16)) return BQ_ERR_ALIGN;
    }
    if (!gemv_chain_eligible(fmt, steps, nsteps, batch)) return BQ_ERR_SHAPE;
    if (!workspace || workspace_bytes < (size_t)bq_gemv_chain_workspace_bytes()) return BQ_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return BQ_ERR_ALIGN;
    const cudaError_t e =
        launch_gemv_chain(fmt, steps, nsteps, batch, static_cast<unsigned int*>(workspace), as_stream(stream));
    return e == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

bq_status bq_check(void* stream) {
    if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return BQ_ERR_CUDA;
    if (cudaGetLastError() != cudaSuccess) return BQ_ERR_CUDA;
    int st = 0;
    if (cudaMemcpyFromSymbol(&st, g_device_status, sizeof(st)) != cudaSuccess) return BQ_ERR_CUDA;
    if (st != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)) != cudaSuccess) return BQ_ERR_CUDA;
        return static_cast<bq_status>(st);
    }
    return BQ_OK;
}

bq_status bq_debug_wait_timeout(int64_t spin_limit, void* stream) {
    if (spin_limit < 0) return BQ_ERR_SHAPE;
    int* flag = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&flag), g_never_set_flag) != cudaSuccess)
        return BQ_ERR_CUDA;
    int* status = device_status_ptr();
    if (!status) return BQ_ERR_CUDA;
    wait_never_set_kernel<<<1, 32, 0, as_stream(stream)>>>(spin_limit, flag, status);
    return cudaGetLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

const char* bq_status_string(int status) {
    switch (status) {
        case BQ_OK: return "ok";
        case BQ_ERR_NULL: return "null pointer";
        case BQ_ERR_SHAPE: return "invalid shape (K % 128 != 0, negative size or batch out of range)";
        case BQ_ERR_ALIGN: return "pointer not aligned as required";
        case BQ_ERR_NONFINITE: return "non-finite weight (NaN or Inf)";
        case BQ_ERR_SCALE_RANGE: return "scale out of FP16 range, negative or non-finite";
        case BQ_ERR_FORMAT: return "unknown format or output dtype";
        case BQ_ERR_CUDA: return "CUDA runtime error";
        case BQ_ERR_TIMEOUT: return "device wait timed out";
        case BQ_ERR_WORKSPACE: return "workspace missing or too small";
        default: return "unknown status";
    }
}

int bq_version(void) { return 100; }

}  // extern "C"
