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
// Eight weights per thread (one 16-byte load, one 4-byte store), so a warp
// reads 512 contiguous bytes; the two (NVFP4) or four (MXFP4) threads of a
// block combine their maxima with shuffles of the bf16 magnitude bits (for
// finite values their integer order is the order of magnitudes).  The NVFP4
// scale is CUDA's saturating round-to-nearest-even E4M3 conversion of the IEEE
// quotient amax/6, and each quotient w/s is an IEEE division.  The MXFP4 scale
// is 2^e with e + 127 = max(exponent field of amax - 2, 0), so w/s is one
// multiplication by 2^-e, exact up to the single rounding the division would
// make.  Each quotient goes to E2M1 by the hardware's round-to-nearest-even,
// saturating conversion, two per instruction, element 2i in the low nibble.
#include "common.cuh"

#include <cuda_fp4.h>
#include <cuda_fp8.h>

namespace w4 {
namespace {

template <int KIND>
__global__ void __launch_bounds__(256) fp4_quant_kernel(const uint4 *__restrict__ W, int64_t N, int64_t K,
                                                        uint32_t *__restrict__ codes, uint8_t *__restrict__ scales)
{
    constexpr int B = KIND == W4_NVFP4 ? 16 : 32;   // weights per block
    constexpr int TPB = B / 8;                       // threads per block
    pdl_wait();
    pdl_launch_dependents();
    const int64_t total = N * (K / 8);               // a multiple of TPB: blocks never straddle rows
    const int lane = threadIdx.x & 31;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    // warp-uniform loop, so that the shuffles see the whole warp
    for (int64_t base = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31); base < total; base += stride) {
        const int64_t t = base + lane;
        const bool valid = t < total;
        const uint4 v = valid ? __ldg(W + t) : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
        uint32_t m = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) m = max(m, max(u[j] & 0x7FFFu, (u[j] >> 16) & 0x7FFFu));
        m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
        if (TPB == 4) m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
        uint8_t scode;
        float sc = 0.f, inv = 0.f;
        if (KIND == W4_NVFP4) {
            const float amax = __uint_as_float(m << 16);
            const __nv_fp8_storage_t f8 = __nv_cvt_float_to_fp8(__fdiv_rn(amax, 6.0f), __NV_SATFINITE, __NV_E4M3);
            scode = (uint8_t)f8;
            sc = __half2float(__half(__nv_cvt_fp8_to_halfraw(f8, __NV_E4M3)));
        } else {
            const int e8 = max((int)(m >> 7) - 2, 0);    // E8M0 code = e + 127
            scode = (uint8_t)e8;
            inv = __uint_as_float((uint32_t)(254 - e8) << 23);   // 2^-e, a normal power of two
        }
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float x0 = bf16lo_to_f32(u[j]), x1 = bf16hi_to_f32(u[j]);
            float2 q;
            if (KIND == W4_NVFP4) q = sc > 0.f ? make_float2(__fdiv_rn(x0, sc), __fdiv_rn(x1, sc)) : make_float2(0.f, 0.f);
            else q = make_float2(x0 * inv, x1 * inv);
            word |= (uint32_t)__nv_cvt_float2_to_fp4x2(q, __NV_E2M1, cudaRoundNearest) << (8 * j);
        }
        if (valid) {
            codes[t] = word;
            if ((lane & (TPB - 1)) == 0) scales[t / TPB] = scode;
        }
    }
}

}  // namespace

cudaError_t launch_fp4_quant(const void *W, int64_t N, int64_t K, int kind, uint8_t *codes, uint8_t *scales,
                             cudaStream_t stream)
{
    const int64_t threads = N * (K / 8);
    const int64_t want = (threads + 255) / 256;
    const unsigned grid = (unsigned)(want < (int64_t)kNumSMs * 16 ? (want > 0 ? want : 1) : (int64_t)kNumSMs * 16);
    if (kind == W4_NVFP4)
        return launch_pdl(fp4_quant_kernel<W4_NVFP4>, dim3(grid), dim3(256), 0, stream, (const uint4 *)W, N, K,
                          (uint32_t *)codes, scales);
    return launch_pdl(fp4_quant_kernel<W4_MXFP4>, dim3(grid), dim3(256), 0, stream, (const uint4 *)W, N, K,
                      (uint32_t *)codes, scales);
}

}  // namespace w4
