// w4_fp4_quant: block-scaled FP4 quantization of a bf16 weight matrix.
//
// Method: page 2 (learn.longtimenohack.com .../quantization.html), the
// Blackwell FP4 paragraph and its teaching snippet: E2M1 values (1 sign, 2
// exponent, 1 mantissa bit), blocks of 16 weights sharing one FP8 E4M3 scale,
// the block's amax mapped to the E2M1 maximum 6 (NVFP4); page 3
// (blog.freezetheflame.cc quantization deep dive) section 4.3: MXFP4, blocks of
// 32 sharing an E8M0 scale, two FP4 values per byte; page 5
// (ai-infra.cypggs.com .../02-core-ideas) section 2.1: the E2M1 value set and
// the E4M3 format.  The exact semantics are spelled out in include/w4.h.
//
// One thread per block: amax over the block's bf16 weights, the scale (E4M3 by
// CUDA's saturating round-to-nearest-even conversion, or the E8M0 power of two
// from the exponent of amax), then per weight the IEEE quotient w / scale
// rounded to E2M1 by comparing its magnitude with the midpoints between
// neighbouring E2M1 values (ties to the even fraction bit), two codes per
// byte.  Consecutive threads take consecutive blocks of a row, so the warp's
// loads and stores are contiguous.
#include "common.cuh"

#include <cuda_fp8.h>

namespace w4 {
namespace {

// E2M1 code of t: nearest of {0, 0.5, 1, 1.5, 2, 3, 4, 6}, ties to the even
// fraction bit (0.25 -> 0, 0.75 -> 1, 1.25 -> 1, 1.75 -> 2, 2.5 -> 2, 3.5 -> 4,
// 5 -> 4), magnitudes above 6 saturating; the sign bit follows t's sign.
__device__ __forceinline__ uint32_t e2m1_code(float t)
{
    const float v = fabsf(t);
    const uint32_t mag = (uint32_t)(v > 0.25f) + (uint32_t)(v >= 0.75f) + (uint32_t)(v > 1.25f) +
                         (uint32_t)(v >= 1.75f) + (uint32_t)(v > 2.5f) + (uint32_t)(v >= 3.5f) + (uint32_t)(v > 5.0f);
    return (signbit(t) ? 8u : 0u) | mag;
}

template <int KIND>
__global__ void __launch_bounds__(256) fp4_quant_kernel(const uint16_t *__restrict__ W, int64_t N, int64_t K,
                                                        uint8_t *__restrict__ codes, uint8_t *__restrict__ scales)
{
    constexpr int B = KIND == W4_NVFP4 ? 16 : 32;   // weights per block
    pdl_wait();
    pdl_launch_dependents();
    const int64_t nb = K / B;                        // blocks per row
    const int64_t total = N * nb;
    for (int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; blk < total;
         blk += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = blk / nb, b = blk - n * nb;
        const uint16_t *w = W + n * K + b * B;
        float x[B];
#pragma unroll
        for (int i = 0; i < B; i += 8) {
            const uint4 v = *(const uint4 *)(w + i);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                x[i + 2 * j] = __uint_as_float(u[j] << 16);
                x[i + 2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
            }
        }
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < B; ++i) amax = fmaxf(amax, fabsf(x[i]));
        float sc;
        uint8_t scode;
        if (KIND == W4_NVFP4) {
            const __nv_fp8_storage_t f8 = __nv_cvt_float_to_fp8(__fdiv_rn(amax, 6.0f), __NV_SATFINITE, __NV_E4M3);
            scode = (uint8_t)f8;
            sc = __half2float(__half(__nv_cvt_fp8_to_halfraw(f8, __NV_E4M3)));
        } else {
            int e = -127;
            if (amax > 0.f) e = min(127, max(-127, ilogbf(amax) - 2));
            scode = (uint8_t)(e + 127);
            sc = ldexpf(1.0f, e);
        }
        scales[n * nb + b] = scode;
        uint32_t packed[B / 8];
#pragma unroll
        for (int i = 0; i < B / 8; ++i) packed[i] = 0u;
#pragma unroll
        for (int i = 0; i < B; ++i) {
            const uint32_t q = sc > 0.f ? e2m1_code(__fdiv_rn(x[i], sc)) : 0u;
            packed[i / 8] |= q << (4 * (i % 8));       // element 2j in the low nibble of byte j
        }
        uint8_t *dst = codes + n * (K / 2) + b * (B / 2);
        if constexpr (B == 16) *(uint2 *)dst = make_uint2(packed[0], packed[1]);
        else *(uint4 *)dst = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
}

}  // namespace

cudaError_t launch_fp4_quant(const void *W, int64_t N, int64_t K, int kind, uint8_t *codes, uint8_t *scales,
                             cudaStream_t stream)
{
    const int64_t B = kind == W4_NVFP4 ? 16 : 32;
    const int64_t total = N * (K / B);
    const int64_t want = (total + 255) / 256;
    const unsigned grid = (unsigned)(want < (int64_t)kNumSMs * 16 ? want : (int64_t)kNumSMs * 16);
    if (kind == W4_NVFP4)
        return launch_pdl(fp4_quant_kernel<W4_NVFP4>, dim3(grid), dim3(256), 0, stream, (const uint16_t *)W, N, K,
                          codes, scales);
    return launch_pdl(fp4_quant_kernel<W4_MXFP4>, dim3(grid), dim3(256), 0, stream, (const uint16_t *)W, N, K, codes,
                      scales);
}

}  // namespace w4
