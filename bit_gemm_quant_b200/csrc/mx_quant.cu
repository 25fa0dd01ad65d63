// w4_mxfp8_quant: MXFP8 activations; w4_mx_scale_layout: E8M0 scales in the
// tensor-core layout; w4_f32_to_bf16: the final rounding of fp32 sums (the
// k-split product reduces fp32 partials before it).
//
// Method: page 3 (blog.freezetheflame.cc quantization deep dive) section 4.3:
// on Blackwell the FP4 weights meet activations kept at FP8, and scales are
// shared by blocks of 32 elements in the E8M0 (power of two) format; page 5
// (ai-infra.cypggs.com .../02-core-ideas) section 2.1 and page 3 section 4.1:
// the E4M3 element format.  The scale exponent is the microscaling rule
// e = floor(log2 amax) - 8 (8 = the exponent of E4M3's largest value 448),
// clamped to [-127, 127]; the exact semantics are spelled out in include/w4.h.
//
// All three kernels are bandwidth-bound elementwise passes.  w4_mxfp8_quant gives one
// thread 8 consecutive elements (one 16-byte load, one 8-byte store); the four
// threads of a 32-element block combine their maxima with two shuffles.  The
// maximum is taken on the bf16 bit patterns without their sign bit (for
// finite values the integer order is the order of magnitudes), so the block's
// E8M0 code is max(exponent field of amax - 8, 0) with no floating point at
// all.  x / 2^e is one multiplication by 2^-e, exact up to the single rounding
// that the IEEE division would also make (2^-e is a normal fp32 power of two
// for every e in range), followed by the hardware's saturating round-to-
// nearest-even E4M3 conversion.
#include "common.cuh"

#include <cuda_fp8.h>

namespace w4 {
namespace {

// Byte offset of the scale of (row r, 32-element block kb) in the tensor-core
// layout of a matrix with K columns: 512-byte atoms of 128 rows x 4 blocks,
// row r of an atom at 16 * (r % 32) + 4 * (r / 32), block kb % 4 in the byte
// of that 32-bit word; atoms ordered by k within a 128-row band.
__host__ __device__ __forceinline__ int64_t mma_sf_offset(int64_t r, int64_t kb, int64_t K)
{
    return (((r >> 7) * (K >> 7) + (kb >> 2)) << 9) + ((r & 31) << 4) + (((r >> 5) & 3) << 2) + (kb & 3);
}

template <int LAYOUT>
__global__ void __launch_bounds__(256) mxfp8_quant_kernel(const uint4 *__restrict__ X, int64_t M, int64_t rows,
                                                          int64_t K, uint2 *__restrict__ codes,
                                                          uint8_t *__restrict__ scales)
{
    pdl_wait();
    pdl_launch_dependents();
    const int64_t per_row = K >> 3;                  // threads per row
    const int64_t total = rows * per_row;            // a multiple of 4: whole 32-element blocks
    const int lane = threadIdx.x & 31;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    // the loop runs warp-uniformly so that the shuffles see the whole warp
    for (int64_t base = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31); base < total; base += stride) {
        const int64_t t = base + lane;
        const bool valid = t < total;
        const int64_t r = valid ? t / per_row : 0;
        const int64_t c8 = valid ? t - r * per_row : 0;
        const bool real = valid && r < M;            // rows >= M only pad the tensor-core layout
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (real) v = __ldg(X + t);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
        uint32_t m = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) m = max(m, max(u[j] & 0x7FFFu, (u[j] >> 16) & 0x7FFFu));
        m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
        const int e8 = max((int)(m >> 7) - 8, 0);   // E8M0 code = e + 127
        const float inv = __uint_as_float((uint32_t)(254 - e8) << 23);   // 2^-e
        uint32_t q[2];
#pragma unroll
        for (int j = 0; j < 4; j += 2) {
            const __nv_fp8x2_storage_t a = __nv_cvt_float2_to_fp8x2(
                make_float2(bf16lo_to_f32(u[j]) * inv, bf16hi_to_f32(u[j]) * inv), __NV_SATFINITE, __NV_E4M3);
            const __nv_fp8x2_storage_t b = __nv_cvt_float2_to_fp8x2(
                make_float2(bf16lo_to_f32(u[j + 1]) * inv, bf16hi_to_f32(u[j + 1]) * inv), __NV_SATFINITE,
                __NV_E4M3);
            q[j / 2] = (uint32_t)a | ((uint32_t)b << 16);
        }
        if (real) codes[t] = make_uint2(q[0], q[1]);
        if (valid && (c8 & 3) == 0) {
            const int64_t kb = c8 >> 2;
            if (LAYOUT == W4_MX_SCALES_MMA) scales[mma_sf_offset(r, kb, K)] = (uint8_t)e8;
            else scales[r * (K >> 5) + kb] = (uint8_t)e8;
        }
    }
}

// dst as uint4 [ceil(R/128)][K/128][32]: element (band, j, l) holds the
// 32-bit words j (blocks 4j..4j+3) of rows band*128 + l + 32i, i = 0..3; rows
// >= R give zero words.
__global__ void __launch_bounds__(256) mx_scale_layout_kernel(const uint32_t *__restrict__ src, int64_t R,
                                                              int64_t K, uint4 *__restrict__ dst)
{
    pdl_wait();
    pdl_launch_dependents();
    const int64_t words = K >> 7;                    // 32-bit words per source row
    const int64_t total = ((R + 127) >> 7) * words * 32;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t l = idx & 31, bj = idx >> 5;
        const int64_t band = bj / words, j = bj - band * words;
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t r = band * 128 + l + 32 * i;
            w[i] = r < R ? __ldg(src + r * words + j) : 0u;
        }
        dst[idx] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// fp32 -> bf16, 4 elements per thread where the pointers allow it
__global__ void __launch_bounds__(256) f32_to_bf16_kernel(const float *__restrict__ src, int64_t n,
                                                          __nv_bfloat16 *__restrict__ dst, int vec)
{
    pdl_wait();
    pdl_launch_dependents();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t t0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (vec) {
        for (int64_t i = t0; i < n / 4; i += stride) {
            const float4 v = __ldg((const float4 *)src + i);
            __nv_bfloat162 *d = (__nv_bfloat162 *)(dst + 4 * i);
            d[0] = __floats2bfloat162_rn(v.x, v.y);
            d[1] = __floats2bfloat162_rn(v.z, v.w);
        }
        for (int64_t i = n / 4 * 4 + t0; i < n; i += stride) dst[i] = __float2bfloat16_rn(src[i]);
    } else {
        for (int64_t i = t0; i < n; i += stride) dst[i] = __float2bfloat16_rn(src[i]);
    }
}

unsigned grid_for(int64_t threads)
{
    const int64_t want = (threads + 255) / 256;
    return (unsigned)(want < (int64_t)kNumSMs * 16 ? (want > 0 ? want : 1) : (int64_t)kNumSMs * 16);
}

}  // namespace

cudaError_t launch_f32_to_bf16(const float *src, int64_t n, void *dst, cudaStream_t stream)
{
    const int vec = ((uintptr_t)src % 16 == 0 && (uintptr_t)dst % 8 == 0) ? 1 : 0;
    return launch_pdl(f32_to_bf16_kernel, dim3(grid_for(vec ? (n + 3) / 4 : n)), dim3(256), 0, stream, src, n,
                      (__nv_bfloat16 *)dst, vec);
}

int64_t mx_padded_rows(int64_t R) { return (R + 127) / 128 * 128; }

cudaError_t launch_mxfp8_quant(const void *X, int64_t M, int64_t K, uint8_t *codes, uint8_t *scales, int layout,
                               cudaStream_t stream)
{
    const int64_t rows = layout == W4_MX_SCALES_MMA ? mx_padded_rows(M) : M;
    const unsigned grid = grid_for(rows * (K / 8));
    if (layout == W4_MX_SCALES_MMA)
        return launch_pdl(mxfp8_quant_kernel<W4_MX_SCALES_MMA>, dim3(grid), dim3(256), 0, stream, (const uint4 *)X, M,
                          rows, K, (uint2 *)codes, scales);
    return launch_pdl(mxfp8_quant_kernel<W4_MX_SCALES_ROWS>, dim3(grid), dim3(256), 0, stream, (const uint4 *)X, M,
                      rows, K, (uint2 *)codes, scales);
}

cudaError_t launch_mx_scale_layout(const uint8_t *src, int64_t R, int64_t K, uint8_t *dst, cudaStream_t stream)
{
    const unsigned grid = grid_for(mx_padded_rows(R) / 128 * (K / 128) * 32);
    return launch_pdl(mx_scale_layout_kernel, dim3(grid), dim3(256), 0, stream, (const uint32_t *)src, R, K,
                      (uint4 *)dst);
}

}  // namespace w4
