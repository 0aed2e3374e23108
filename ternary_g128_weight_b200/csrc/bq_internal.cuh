// Internal declarations shared by the library's translation units.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "bq.h"

namespace bq {

constexpr int kGroup = 128;

// Device-side status words live in bq_api.cu; kernels receive their
// addresses as arguments.
//   status      : first error of a bounded device wait that gave up.
//   pack_first  : first failing group of a packer call, encoded
//                 (group index << 8) | status, so that the error reported is the
//                 one of the lowest (row, group) as in the sequential
//                 definition; ~0 means none.
__device__ __forceinline__ void record_status(int* status, int st) {
    atomicCAS(status, 0, st);
}

__device__ __forceinline__ void record_pack_error(unsigned long long* first, int64_t group_index, int st) {
    atomicMin(first, ((unsigned long long)group_index << 8) | (unsigned)st);
}

// Address of the device status word of the current device.
int* device_status_ptr();

// Per-device launcher state (bq_device.cu): the current device's SM count,
// raising a kernel's opt-in dynamic shared memory on the current device (once
// per kernel and device), and the driver's cuTensorMapEncodeTiled (NULL if the
// driver lacks it).  Safe to call from several host threads.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
int sm_count();
cudaError_t ensure_dynamic_smem(const void* func, int bytes);
EncodeTiledFn encode_fn();

// Low / high BF16 of a packed pair -> float.
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ float half_bits_to_float(uint16_t h) {
    return __half2float(__ushort_as_half(h));
}

__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Host-side launchers (return cudaGetLastError() of the launch).
cudaError_t launch_pack(int fmt, const float* w, int64_t n, int64_t k, const uint16_t* scales_in,
                        uint8_t* codes, uint16_t* scales, unsigned long long* first_error,
                        cudaStream_t s);
cudaError_t launch_wait_timeout(int64_t spin_limit, cudaStream_t s);

// Tensor-core decode GEMV (binary and 2-bit ternary, batch <= 4, K % 1024 == 0).
bool gemv_tc_eligible(int fmt, int64_t n, int64_t k, int batch);
int64_t gemv_tc_workspace_bytes(int fmt, int64_t n, int64_t k, int batch);
cudaError_t launch_gemv_tc(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                           const uint16_t* x, int batch, void* y, int y_dtype, void* workspace, cudaStream_t s);

// Row-owning decode GEMV (all three formats, batch <= 8, K % 1024 == 0,
// activation operand resident in shared memory): no workspace.
bool gemv_rows_eligible(int fmt, int64_t n, int64_t k, int batch);
cudaError_t launch_gemv_rows(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                             const uint16_t* x, int batch, void* y, int y_dtype, cudaStream_t s);

// Wide-batch decode GEMV (binary and 2-bit ternary, batch 5..16, K % 1024 ==
// 0, FP16 activations of all of K resident in shared memory): no workspace.
bool gemv_wide_eligible(int fmt, int64_t n, int64_t k, int batch);
cudaError_t launch_gemv_wide(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                             const uint16_t* x, int batch, void* y, int y_dtype, cudaStream_t s);

// Embedding lookup (bq_embed_rows).
cudaError_t launch_embed_rows(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                              const int32_t* ids, int64_t count, uint16_t* out, cudaStream_t s);

// Persistent layer chain (bq_gemv_chain): eligibility of the step list and
// its launch; bar = the two zeroed barrier counters.
bool gemv_chain_eligible(int fmt, const bq_chain_step* steps, int nsteps, int batch);
cudaError_t launch_gemv_chain(int fmt, const bq_chain_step* steps, int nsteps, int batch, unsigned int* bar,
                              cudaStream_t s);

// GEMV path choice shared by bq_gemv, bq_gemm (T <= 16) and bq_gemv_noalloc:
// batch 5..16 the wide-batch kernel where eligible; the row-owning kernel
// where eligible, else the split-K tensor-core kernel,
// else the tcgen05 GEMM with T = batch; None when no kernel takes the shape
// (K > 2^28 or N >= 2^31).  gemv_workspace_bytes reports the workspace of the
// choice.
enum class GemvPath { Rows, Wide, SplitK, Gemm, None };
GemvPath gemv_path(int fmt, int64_t n, int64_t k, int batch);
int64_t gemv_workspace_bytes(int fmt, int64_t n, int64_t k, int batch);
cudaError_t launch_gemv(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                        const uint16_t* x, int batch, void* y, int y_dtype, void* workspace, cudaStream_t s);

// tcgen05 prefill GEMM (all formats, K % 128 == 0).
bool gemm_tc_eligible(int fmt, int64_t n, int64_t k, int64_t t);
int64_t gemm_tc_workspace_bytes(int64_t n, int64_t k, int64_t t);
int gemm_tc_launches(int64_t n, int64_t k, int64_t t);
cudaError_t launch_gemm_tc(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t n, int64_t k,
                           const uint16_t* x, int64_t t, void* y, int y_dtype, void* workspace, cudaStream_t s);

}  // namespace bq
