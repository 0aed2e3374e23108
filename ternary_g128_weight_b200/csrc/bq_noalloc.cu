// bq_gemv_noalloc: the GEMV for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they run a product:
// a host framework that owns all device memory and hands a plugin only its
// input and output buffers, or a latency-critical path where cudaMalloc (which
// may synchronise the device) is not allowed.  bq_gemv needs a caller-provided
// workspace for its tensor-core path; this entry point instead uses one fixed
// scratch array that lives in the library's device image, so the caller passes
// only codes, scales, x and y.
//
// The scratch array is BQ_NOALLOC_SCRATCH_BYTES bytes, a file-scope __device__
// variable: every GPU that loads the library holds it until the process exits.
// Host code must not use the symbol `g_noalloc_scratch` as an address (in
// host code it is only a stand-in for the device variable); the device address
// is looked up once per device with cudaGetSymbolAddress, with that device
// current, on the first call made on it.  All calls share the array and it
// keeps the last call's contents; the kernels clear what must start at zero
// (the split-K row-block counters) on every call.  Two calls that overlap on
// the GPU (different streams, no ordering between them) race on the array.
#include <mutex>

#include "bq_internal.cuh"

static __device__ __align__(256) uint8_t g_noalloc_scratch[BQ_NOALLOC_SCRATCH_BYTES];

namespace bq {
namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
uint8_t* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
bq_status noalloc_scratch(uint8_t** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return BQ_ERR_CUDA;
        g_noalloc_ptr[dev] = static_cast<uint8_t*>(p);
    }
    *out = g_noalloc_ptr[dev];
    return BQ_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace bq

using namespace bq;

extern "C" bq_status bq_gemv_noalloc(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                                     const uint16_t* x, int batch, void* y, int y_dtype, void* stream) {
    if (fmt != BQ_Q1G128 && fmt != BQ_T2G128 && fmt != BQ_T5P8G128 && fmt != BQ_A1G128) return BQ_ERR_FORMAT;
    if (n < 0 || k < 0 || k % kGroup != 0 || batch < 1 || batch > BQ_MAX_BATCH) return BQ_ERR_SHAPE;
    if (y_dtype != BQ_BF16 && y_dtype != BQ_F32) return BQ_ERR_FORMAT;
    if (n == 0) return BQ_OK;
    if (!y || (k > 0 && (!codes || !scales || !x))) return BQ_ERR_NULL;
    if (!aligned16(y) || (k > 0 && (!aligned16(codes) || !aligned16(scales) || !aligned16(x)))) return BQ_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (k == 0) {
        const size_t bytes = (size_t)batch * n * (y_dtype == BQ_F32 ? 4 : 2);
        return cudaMemsetAsync(y, 0, bytes, s) == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
    }
    // Same path choice as bq_gemv.  The row-owning and wide-batch kernels
    // need no scratch; the split-K kernel keeps its prepared activations,
    // row-block counters and partial sums there, and the tcgen05 GEMM
    // (T = batch) its FP16 activations, per-token scales and, when K is split,
    // partial tiles.
    if (gemv_path(fmt, n, k, batch) == GemvPath::None) return BQ_ERR_SHAPE;
    const int64_t need = gemv_workspace_bytes(fmt, n, k, batch);
    uint8_t* scratch = nullptr;
    if (need > 0) {
        if (need > (int64_t)BQ_NOALLOC_SCRATCH_BYTES) return BQ_ERR_WORKSPACE;
        const bq_status st = noalloc_scratch(&scratch);
        if (st != BQ_OK) return st;
    }
    const cudaError_t e = launch_gemv(fmt, codes, scales, n, k, x, batch, y, y_dtype, scratch, s);
    return e == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}
