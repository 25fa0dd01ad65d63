// Shared helpers of libw4 (CUDA side only).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "w4.h"

namespace w4 {

constexpr int kNumSMs = 148;             // B200

__device__ __forceinline__ float bf16lo_to_f32(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Launchers (host side), implemented in the kernel files.
cudaError_t launch_quant_pack(const void *W, int64_t N, int64_t K, int group, int mode, const float *s,
                              uint32_t *qweight, void *scales, uint32_t *qzeros, cudaStream_t stream);
cudaError_t launch_gemv(const void *X, int64_t M, int64_t N, int64_t K, const uint32_t *qweight,
                        const void *scales, const uint32_t *qzeros, int group, int mode, void *Y,
                        cudaStream_t stream);
size_t tc_workspace_bytes(int64_t M, int64_t N, int64_t K);
cudaError_t launch_gemm_tc(const void *X, int64_t M, int64_t N, int64_t K, const uint32_t *qweight,
                           const void *scales, const uint32_t *qzeros, int group, int mode, void *Y, void *ws,
                           cudaStream_t stream);
int read_and_clear_device_error();

}  // namespace w4
