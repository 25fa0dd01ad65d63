// w4a16_gemm, M <= 8: the decode GEMV / skinny path.
//
// Method: page 2 (learn.longtimenohack.com .../quantization.html) opens with
// "reading weights is the top cost of decode", page 4
// (llm-glossary.tokens-kit.com/terms/quantization-methods/, GPTQ section) with
// "small-batch decode profits from the weight bandwidth", and page 3
// (blog.freezetheflame.cc quantization deep dive) section 1.2 with "fuse
// dequantize into the GEMM so the weights stay 4-bit in HBM"; section 3.1 of
// the same page sketches Marlin, which unpacks INT4 in registers and feeds
// mma.sync.  Dequantization follows page 5 (ai-infra.cypggs.com
// .../02-core-ideas) section 2.2, x^ = (q - zp) * s, rounded once to bf16.
//
// Design (HBM-bound: 0.5 B of codes + 1/64 B of scale per weight at g = 128):
//   * a CTA (4 warps) owns a tile of 16 output channels and all of K; its
//     warps split K into 512-wide super-chunks (warp w takes super-chunks w,
//     w+4, ...) and sum their partial tiles in shared memory at the end (no
//     global scratch); small CTAs keep many tiles resident per SM;
//   * at launch the CTA's first threads ask L2 to fetch the tile's codes,
//     scales and zero-points (cp.async.bulk.prefetch, one instruction per
//     channel), so every byte of the tile is requested from HBM at once and
//     the warps' own loads see L2 latency; small CTAs keep several tiles per
//     SM in flight;
//   * lane (g, t) = (lane/4, lane%4) of a warp loads, for channels g and g+8,
//     the 64 contiguous bytes (128 codes) at k = 512*sc + 128*t, with the
//     scales and zero-points of their groups, and the activations one 32-wide
//     step ahead;
//   * each 32-bit word of codes gives four bf16x2 pairs of ADJACENT elements
//     with one shift and one LOP3 (the packed layout keeps even elements in
//     the low half-word), as 128 + u via the bf16 exponent of 128;
//   * exact w^ = bf16_rne((u - zp) * s16) with three bf16x2 operations:
//     D = (128+u) - (128+zp) (exact), c = D * s_lo (exact: <= 7 bits) and
//     w^ = fma(D, s_hi, c), where s16 = s_hi + s_lo splits the fp16 scale into
//     its bf16 rounding and the (<= 3-bit) remainder; the fused multiply-add
//     rounds the exact product D * s16 once;
//   * mma.sync m16n8k16 (bf16 in, fp32 accumulate) takes those registers as
//     its A fragment directly: the k-order inside an MMA is free, so a
//     thread's logical columns (2t, 2t+1) and (2t+8, 2t+9) are mapped to the
//     physical elements 8w+4h+{0,1} and 8w+4h+{2,3} of its own words, and the
//     activation fragment for token g is then the plain 16-byte chunk
//     X[g][k + 8w .. k + 8w + 7];
//   * tokens occupy the MMA's N = 8 columns; lanes with g >= M feed zeros.
#include "common.cuh"

namespace w4 {
namespace {

__device__ __forceinline__ uint32_t bf2_sub(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t bf2_mul(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t bf2_fma(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t d;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Per-(channel, group) dequantization constants, each duplicated into both
// halves of a bf16x2: s_hi = bf16_rne(s16), s_lo = s16 - s_hi, Z = 128 + zp.
struct GroupConst {
    uint32_t shi, slo, z;
};

__device__ __forceinline__ GroupConst group_const(unsigned short s16bits, int zp)
{
    const float sf = __half2float(__ushort_as_half(s16bits));
    const __nv_bfloat16 hi = __float2bfloat16_rn(sf);
    const __nv_bfloat16 lo = __float2bfloat16_rn(sf - __bfloat162float(hi));   // exact
    const uint32_t h = __bfloat16_as_ushort(hi), l = __bfloat16_as_ushort(lo);
    GroupConst gc;
    gc.shi = h | (h << 16);
    gc.slo = l | (l << 16);
    gc.z = 0x43004300u | ((uint32_t)zp << 16) | (uint32_t)zp;
    return gc;
}

// w^ for elements (8c+2j, 8c+2j+1) of packed word q.
__device__ __forceinline__ uint32_t dequant_pair(uint32_t q, int j, const GroupConst &gc)
{
    const uint32_t v = ((q >> (4 * j)) & 0x000F000Fu) | 0x43004300u;   // 128 + u, as bf16x2
    const uint32_t D = bf2_sub(v, gc.z);
    return bf2_fma(D, gc.shi, bf2_mul(D, gc.slo));
}

constexpr int kWarps = 4;

template <int G, int MODE>
__global__ void __launch_bounds__(kWarps * 32)
gemv_kernel(const uint4 *__restrict__ X, int M, int N, int K, const uint4 *__restrict__ qweight,
            const unsigned short *__restrict__ scales, const uint32_t *__restrict__ qzeros,
            __nv_bfloat16 *__restrict__ Y)
{
    constexpr int QPG = G / 32;                  // 16-byte code chunks per group
    constexpr int NGI = 4 / QPG;                 // groups per super-chunk and channel, per lane
    __shared__ float red[kWarps][32][4];

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int KQ = K >> 5;                       // 16-byte code chunks per channel
    const int NG = K / G, ZW = (NG + 7) >> 3;
    const int r0 = (int)blockIdx.x * 16;
    const int rA = r0 + g, rB = rA + 8;
    const bool okA = rA < N, okB = rB < N;
    const int rows = min(16, N - r0);

    // the whole tile, HBM -> L2, before any thread waits on a load
    if (threadIdx.x < rows) prefetch_l2(qweight + (size_t)(r0 + threadIdx.x) * KQ, (size_t)KQ * 16);
    else if (threadIdx.x == 16) prefetch_l2(scales + (size_t)r0 * NG, (size_t)rows * NG * 2);
    else if (threadIdx.x == 17 && MODE == W4_ASYM) prefetch_l2(qzeros + (size_t)r0 * ZW, (size_t)rows * ZW * 4);

    const bool has_x = g < M;
    const uint4 *xrow = X + (size_t)(has_x ? g : 0) * (K >> 3);
    const uint4 *qa = qweight + (size_t)(okA ? rA : 0) * KQ;
    const uint4 *qb = qweight + (size_t)(okB ? rB : 0) * KQ;
    const unsigned short *sa_row = scales + (size_t)(okA ? rA : 0) * NG;
    const unsigned short *sb_row = scales + (size_t)(okB ? rB : 0) * NG;
    const uint32_t *za_row = qzeros + (size_t)(okA ? rA : 0) * ZW;
    const uint32_t *zb_row = qzeros + (size_t)(okB ? rB : 0) * ZW;

    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    // warp w takes the 512-wide super-chunks w, w+4, ...; lane t their chunks 4t..4t+3
    for (int s0 = warp * 16; s0 < KQ; s0 += kWarps * 16) {
        const int q0 = s0 + 4 * t;
        uint4 a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const bool ok = q0 + i < KQ;
            a[i] = (ok && okA) ? __ldg(qa + q0 + i) : make_uint4(0u, 0u, 0u, 0u);
            b[i] = (ok && okB) ? __ldg(qb + q0 + i) : make_uint4(0u, 0u, 0u, 0u);
        }
        unsigned short sa[NGI], sb[NGI];
        uint32_t za[NGI], zb[NGI];
#pragma unroll
        for (int u = 0; u < NGI; ++u) {
            const int qi = q0 + u * QPG;
            const bool ok = qi < KQ;
            const int j = ok ? (qi * 32) / G : 0;
            sa[u] = (ok && okA) ? __ldg(sa_row + j) : (unsigned short)0;
            sb[u] = (ok && okB) ? __ldg(sb_row + j) : (unsigned short)0;
            if (MODE == W4_ASYM) {
                za[u] = (ok && okA) ? (__ldg(za_row + (j >> 3)) >> (4 * (j & 7))) & 0xFu : 0u;
                zb[u] = (ok && okB) ? (__ldg(zb_row + (j >> 3)) >> (4 * (j & 7))) & 0xFu : 0u;
            } else {
                za[u] = zb[u] = 8u;
            }
        }
        uint4 xv[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) xv[w] = (has_x && q0 < KQ) ? __ldg(xrow + q0 * 4 + w) : make_uint4(0u, 0u, 0u, 0u);
        GroupConst ca, cb;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int qi = q0 + i;
            uint4 xn[4];                         // activations of the next 32-wide step
            const bool okn = has_x && i < 3 && qi + 1 < KQ;
#pragma unroll
            for (int w = 0; w < 4; ++w) xn[w] = okn ? __ldg(xrow + (qi + 1) * 4 + w) : make_uint4(0u, 0u, 0u, 0u);
            if (i % QPG == 0) {
                ca = group_const(sa[i / QPG], (int)za[i / QPG]);
                cb = group_const(sb[i / QPG], (int)zb[i / QPG]);
            }
            const uint32_t wa[4] = {a[i].x, a[i].y, a[i].z, a[i].w};
            const uint32_t wb[4] = {b[i].x, b[i].y, b[i].z, b[i].w};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const uint32_t a0 = dequant_pair(wa[w], 0, ca), a1 = dequant_pair(wa[w], 1, ca);
                const uint32_t a2 = dequant_pair(wa[w], 2, ca), a3 = dequant_pair(wa[w], 3, ca);
                const uint32_t b0 = dequant_pair(wb[w], 0, cb), b1 = dequant_pair(wb[w], 1, cb);
                const uint32_t b2 = dequant_pair(wb[w], 2, cb), b3 = dequant_pair(wb[w], 3, cb);
                mma_bf16_16816(acc, a0, b0, a1, b1, xv[w].x, xv[w].y);
                mma_bf16_16816(acc, a2, b2, a3, b3, xv[w].z, xv[w].w);
            }
#pragma unroll
            for (int w = 0; w < 4; ++w) xv[w] = xn[w];
        }
    }

#pragma unroll
    for (int i = 0; i < 4; ++i) red[warp][lane][i] = acc[i];
    __syncthreads();
    if (warp == 0) {
        float sm[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int w = 0; w < kWarps; ++w)
#pragma unroll
            for (int i = 0; i < 4; ++i) sm[i] += red[w][lane][i];
        const int m0 = 2 * t, m1 = 2 * t + 1;    // tokens of c0/c2 and c1/c3
        if (okA && m0 < M) Y[(size_t)m0 * N + rA] = __float2bfloat16_rn(sm[0]);
        if (okA && m1 < M) Y[(size_t)m1 * N + rA] = __float2bfloat16_rn(sm[1]);
        if (okB && m0 < M) Y[(size_t)m0 * N + rB] = __float2bfloat16_rn(sm[2]);
        if (okB && m1 < M) Y[(size_t)m1 * N + rB] = __float2bfloat16_rn(sm[3]);
    }
}

template <int G, int MODE>
cudaError_t launch_g_mode(const void *X, int64_t M, int64_t N, int64_t K, const uint32_t *qweight,
                          const void *scales, const uint32_t *qzeros, void *Y, cudaStream_t stream)
{
    const int64_t blocks = (N + 15) / 16;       // one 16-channel tile per CTA
    gemv_kernel<G, MODE><<<(unsigned)blocks, kWarps * 32, 0, stream>>>(
        (const uint4 *)X, (int)M, (int)N, (int)K, (const uint4 *)qweight, (const unsigned short *)scales, qzeros,
        (__nv_bfloat16 *)Y);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemv(const void *X, int64_t M, int64_t N, int64_t K, const uint32_t *qweight,
                        const void *scales, const uint32_t *qzeros, int group, int mode, void *Y,
                        cudaStream_t stream)
{
    switch (group * 2 + mode) {
    case 32 * 2 + W4_SYM: return launch_g_mode<32, W4_SYM>(X, M, N, K, qweight, scales, qzeros, Y, stream);
    case 32 * 2 + W4_ASYM: return launch_g_mode<32, W4_ASYM>(X, M, N, K, qweight, scales, qzeros, Y, stream);
    case 64 * 2 + W4_SYM: return launch_g_mode<64, W4_SYM>(X, M, N, K, qweight, scales, qzeros, Y, stream);
    case 64 * 2 + W4_ASYM: return launch_g_mode<64, W4_ASYM>(X, M, N, K, qweight, scales, qzeros, Y, stream);
    case 128 * 2 + W4_SYM: return launch_g_mode<128, W4_SYM>(X, M, N, K, qweight, scales, qzeros, Y, stream);
    case 128 * 2 + W4_ASYM: return launch_g_mode<128, W4_ASYM>(X, M, N, K, qweight, scales, qzeros, Y, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace w4
