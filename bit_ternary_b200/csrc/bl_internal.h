// bl_internal.h - declarations shared by the libbitlinear translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bl_device.cuh"

namespace bl {

// Pack workspace: header (status word at 0, mean_c and s at 16/20) + 256 bins.
constexpr size_t kPackWsBytes = kHeaderBytes + 256 * sizeof(unsigned long long);

// Largest shared-memory footprint of the fused quantise + GEMV kernel for the
// quantised activations; above it the forward takes the tensor-core path.
constexpr int64_t kGemvMaxM = 16;
constexpr int64_t kGemvMaxSmemQ = 160 * 1024;

inline int64_t gemv_q_stride(int64_t K) { return ((K + 255) / 256) * 256 + 16; }
inline bool gemv_eligible(int64_t M, int64_t K) {
  return M <= kGemvMaxM && M * gemv_q_stride(K) <= kGemvMaxSmemQ;
}

cudaError_t launch_pack(const float* W, int64_t N, int64_t K, uint32_t* packed, float* D, void* ws,
                        cudaStream_t stream, int num_sms);
// err_reset (nullable): the workspace error word, cleared by the kernel.
cudaError_t launch_act_quant(const float* x, int64_t M, int64_t K, int8_t* q, float* s_x, int32_t* rowsum,
                             bool permuted, cudaStream_t stream, uint32_t* err_reset);
cudaError_t launch_gemv(const float* x, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                        const float* D, float* y, int32_t* acc_out, uint32_t* err_reset, cudaStream_t stream,
                        int num_sms);
// Expects the permuted activations, s_x and row sums already in the forward
// workspace (launch_act_quant with permuted = true).
cudaError_t launch_gemm(int64_t M, int64_t N, int64_t K, const uint32_t* packed, const float* D, float* y,
                        int32_t* acc_out, void* ws, cudaStream_t stream, int num_sms);

cudaError_t launch_selftest_wait(uint32_t* err, uint64_t limit_ns, cudaStream_t stream);

}  // namespace bl
